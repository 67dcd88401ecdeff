/*
 * bs.h -- C ABI of libbs, the B200 (sm_100a) decoder for BF16RANS containers.
 *
 * The method is the one the "Qwen3.8-27B-BF16-NVLC-Lossless" model card describes in the
 * paragraph after its accounting table:
 *   - each BF16 word is split into sign:1 | exponent:8 | fraction:7;
 *   - the joint sign+exponent symbol is rANS-coded with a per-tensor model;
 *   - the decoded symbol selects the distribution of the 7-bit fraction (here a table over
 *     its top three bits; the low four bits are kept verbatim);
 *   - the fields are recombined bitwise, so the output is byte-identical to the original.
 * The container (BF16RANS version 2: interleaved 32-lane chunks, quantised tables, raw
 * spans, a per-tensor checksum) is this library's own design; the card gives no byte layout.
 * Each declaration below names the passage that defines its operation, or says that it is
 * this library's design.
 *
 * Conventions
 *  - Every function returns a bs_status, and nothing throws across the ABI.
 *  - The caller owns every device buffer: the container copy, the workspace and the
 *    outputs. The library allocates no device memory. Its only allocation is host memory
 *    inside a plan, which bs_plan_destroy frees.
 *  - "stream" is a cudaStream_t passed as void*, so that this header needs no CUDA
 *    header. 0 means the legacy default stream.
 *  - A plan is immutable after bs_plan returns. Decodes of the same plan may run
 *    concurrently on different streams into disjoint outputs. They share the plan's
 *    device error word, which records corruption found by any of them.
 *  - Corruption found on the device is reported asynchronously through bs_check.
 *    Kernels never trap, and every device loop is bounded by the chunk's weight count.
 */
#ifndef BS_H
#define BS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BS_OK = 0,
    BS_E_ARG = 1,          /* null pointer, bad index, misaligned buffer, bad size */
    BS_E_FORMAT = 2,       /* the container fails validation (bad magic, offsets, tables, sizes) */
    BS_E_VERSION = 3,      /* unknown magic version */
    BS_E_SIZE = 4,         /* an output or workspace buffer is the wrong size */
    BS_E_CUDA = 5,         /* a CUDA runtime call failed (the CUDA error is kept, see bs_last_cuda_error) */
    BS_E_CORRUPT = 6,      /* a chunk failed its end check, or a checksum differs */
    BS_E_NOMEM = 7,        /* host allocation failed */
    BS_E_UNSUPPORTED = 8   /* a device without sm_100 support */
} bs_status;

enum { BS_KIND_RANS = 0, BS_KIND_STORED = 1, BS_KIND_RAW = 2, BS_KIND_JOINT = 3 };

typedef struct bs_plan_t bs_plan_t; /* opaque host object */

typedef struct {
    uint64_t n_elems;     /* weights (RANS, STORED) or bytes (RAW) */
    uint64_t out_bytes;   /* size of the decoded tensor: 2*n_elems, or n_elems for RAW */
    uint64_t coded_bytes; /* RANS: model + chunk table + chunk payloads (padded); else out_bytes */
    uint64_t n_chunks;    /* RANS only */
    uint64_t checksum;    /* of the original tensor: sum of splitmix64((i << 16) | w[i]) mod 2^64 */
    uint64_t shape[8];
    uint32_t kind;        /* BS_KIND_* */
    uint32_t ndim;
    uint32_t ns, nh, n_routes, log2_chunk; /* RANS: s-table and h-table precisions, routes, chunk; JOINT: ns = nj, nh = n_routes = 0 */
    const char* name;     /* not NUL-terminated; points into the plan */
    uint32_t name_bytes;
    uint32_t nib_mode;    /* RANS: 0 = nibbles stored, 0x10 + c = every low nibble is c */
} bs_tensor_info;

/* Bytes of device workspace that bs_plan needs for this container: the decode
 * tables of every coded tensor plus a 256-byte error block. h_container must hold the
 * whole container. Returns 0 if the container does not validate. This library's design. */
size_t bs_plan_workspace_bytes(const void* h_container, size_t container_bytes);

/*
 * bs_plan: parse and validate a container, build its decode tables and upload them.
 * Source: the per-tensor model of the NVLC card's field-split paragraph (each tensor carries
 * its own quantised frequency tables; here they are expanded into slot tables for the
 * decode). Validation, the workspace and the plan object are this library's design.
 *
 *   h_container      host copy of the whole container (read only during the call), or
 *                    NULL: the plan then reads the header, directory, models and chunk
 *                    tables from d_container with synchronous copies on stream
 *   container_bytes  its length, equal to the header's total_bytes
 *   d_container      the same bytes in device memory, 16-byte aligned; it must stay
 *                    alive and unchanged for the life of the plan
 *   d_workspace      device buffer of at least bs_plan_workspace_bytes, 256-byte aligned;
 *                    the plan owns its contents until bs_plan_destroy
 *   stream           the tables are uploaded with cudaMemcpyAsync on this stream
 *   out              receives the plan
 *
 * Validation checks every offset, size, table sum and start state before any device work: a
 * bad container gives BS_E_FORMAT or BS_E_VERSION, and a short workspace gives BS_E_SIZE.
 */
bs_status bs_plan(const void* h_container, size_t container_bytes, const void* d_container, void* d_workspace,
                  size_t workspace_bytes, void* stream, bs_plan_t** out);

/* As bs_plan_workspace_bytes, reading the metadata from device memory (synchronous
 * copies on stream). Returns 0 if the container does not validate. This library's design. */
size_t bs_plan_workspace_bytes_device(const void* d_container, size_t container_bytes, void* stream);

/* Frees the plan's host memory. The caller's device buffers are untouched. */
void bs_plan_destroy(bs_plan_t* plan);

/* The directory as parsed (this library's design): tensor count, and one entry's metadata.
 * BS_E_ARG for a NULL pointer or an index out of range. */
bs_status bs_tensor_count(const bs_plan_t* plan, int32_t* n);
bs_status bs_tensor_info_get(const bs_plan_t* plan, int32_t idx, bs_tensor_info* out);

/*
 * bs_decode_tensor: decode tensor idx into d_out (device, 16-byte aligned, out_bytes =
 * the tensor's out_bytes; otherwise BS_E_SIZE / BS_E_ARG). The work is enqueued on stream
 * and the call returns at once.
 * Source: the NVLC card's field-split paragraph. The sign+exponent symbol is rANS-decoded
 * with the tensor's model, it selects the fraction's distribution, the fraction is decoded
 * with it, and the fields are recombined bitwise into the original word; non-BF16 spans come
 * back verbatim from the residual stream. The 32 interleaved lanes per chunk are this
 * library's reading of the card's "lane-oriented streams" (runtime streams paragraph).
 *  - RANS and JOINT: the interleaved rANS decode kernel, with one warp-lane per rANS state.
 *  - STORED and RAW: a vectorised copy kernel.
 */
bs_status bs_decode_tensor(const bs_plan_t* plan, int32_t idx, void* d_out, size_t out_bytes, void* stream);

/*
 * bs_decode_batch: decode n tensors in one pass: the operation of bs_decode_tensor for each.
 * The batching is this library's design. All the coded tensors of one kernel instance go in a
 * single launch (more than 500 of them are split across launches), and STORED/RAW tensors in
 * one copy launch. idx[k] goes to d_out[k], of out_bytes[k] bytes.
 *  - The outputs must not overlap.
 *  - idx, d_out and out_bytes are host arrays, read during the call.
 */
bs_status bs_decode_batch(const bs_plan_t* plan, const int32_t* idx, void* const* d_out, const size_t* out_bytes,
                          int32_t n, void* stream);

/*
 * bs_decode_ranges: decode parts of tensors, in whole chunks, in one pass (the launches of
 * bs_decode_batch). It serves callers that decode a checkpoint in batches of a fixed size,
 * say 1 GB of output at a time, where one batch may end inside a tensor and the next one
 * continue it. The operation is bs_decode_tensor's; cutting at chunk boundaries is this
 * library's design.
 *  - Range k decodes elements [begin, begin + count) of tensor idx (bytes for RAW) into
 *    d_out, which receives exactly those words: out_bytes = 2 * count (RAW: count).
 *  - RANS and JOINT tensors: begin must be a multiple of the tensor's chunk size
 *    (2^log2_chunk) and the range must end on a chunk boundary or at the tensor's end,
 *    else BS_E_ARG. d_out must then be 16-byte aligned. STORED and RAW ranges, and empty
 *    ranges of any kind, may start and end anywhere inside the tensor.
 *  - A range past the tensor's end, a negative or unknown idx or a nonzero reserved field
 *    gives BS_E_ARG; a wrong out_bytes gives BS_E_SIZE. Nothing is launched then.
 *  - Outputs must not overlap. ranges is a host array, read during the call.
 *  - A corrupt chunk is reported by bs_check with the tensor's own chunk index.
 */
typedef struct {
    int32_t idx;        /* tensor */
    uint32_t reserved;  /* 0 */
    uint64_t begin;     /* first element (RAW: byte) */
    uint64_t count;     /* elements (RAW: bytes) */
    void* d_out;        /* device, caller-owned */
    size_t out_bytes;
} bs_range;

bs_status bs_decode_ranges(const bs_plan_t* plan, const bs_range* ranges, int32_t n, void* stream);

/*
 * bs_decode_geometry: how the decode kernel splits tensor idx on the current device, for
 * callers that cut their decode into batches (bs_decode_ranges). This library's design.
 *  - *chunks_per_cta receives the chunks one CTA takes at the kernel's largest shape. All of
 *    a CTA's chunks come from one tensor, so a range whose chunk count is not a multiple of
 *    it leaves its last CTA part-filled. STORED and RAW tensors give 0.
 *  - *ctas_per_wave receives the CTAs that run at once on the device: one per SM.
 * A launch of more CTAs than one wave runs in several waves, and a last wave with few CTAs
 * costs as much time as a full one. A batch whose ranges take at most ctas_per_wave CTAs
 * (each range taking ceil(chunks / chunks_per_cta)) runs as a single wave.
 * Returns BS_E_ARG for a bad idx or a NULL output pointer, BS_E_CUDA if the device cannot
 * be queried.
 */
bs_status bs_decode_geometry(const bs_plan_t* plan, int32_t idx, uint32_t* chunks_per_cta, uint32_t* ctas_per_wave);

/*
 * bs_verify_tensor: compute the per-tensor checksum (sum over i of splitmix64((i << 16) |
 * w[i]) mod 2^64; bytes for RAW) of a decoded tensor on the device and compare it with the
 * stored one. The check is the analogue of the per-tensor
 * md5 that the "Gemma 2 9B Instruct -- Lossless Compressed" card ("What lossless
 * means") runs at decompression.
 *  - d_scratch: 16 device bytes, 8-byte aligned, owned by the caller.
 *  - Synchronises stream. Returns BS_E_CORRUPT on a mismatch.
 *  - *got may be NULL. Otherwise it receives the computed checksum.
 */
bs_status bs_verify_tensor(const bs_plan_t* plan, int32_t idx, const void* d_out, size_t out_bytes,
                           void* d_scratch, void* stream, uint64_t* got);

/*
 * bs_check: synchronise stream, then read and clear the plan's device error word. The check
 * behind it is this library's design: every rANS lane of a chunk must end in the state L the
 * encoder started from, having consumed exactly the chunk's words.
 * Returns BS_E_CORRUPT if any decode since the last check found a corrupt chunk. In
 * that case *first_bad (if not NULL) is (tensor_index << 40) | chunk_index of the
 * smallest such pair, and -1 otherwise.
 */
bs_status bs_check(const bs_plan_t* plan, void* stream, int64_t* first_bad);

/*
 * bs_decode_tensor_noalloc: decode one tensor with no device memory from the caller beyond
 * the container and the output. The paper has no counterpart: this is a convenience of
 * this library.
 *
 * For callers that cannot allocate device memory: for example a plugin inside another
 * runtime whose allocator owns all of the GPU's memory, or a callback where an allocation
 * would synchronise the device or is not allowed.
 *
 * Instead of a caller workspace, the decode tables (at most 64 KiB) and the error block live
 * in a static device array of 64 KiB + 256 bytes. Every GPU that loads libbs holds that array
 * until the process exits.
 *
 *   h_container      host copy of the whole container; tensor idx is validated in place
 *                    (no host allocation)
 *   d_container      the same bytes on the device, 16-byte aligned
 *   d_out, out_bytes as for bs_decode_tensor
 *
 * Behaviour:
 *  - The first call on a device looks up the array's device address with
 *    cudaGetSymbolAddress. Make that first call before any stream capture.
 *  - Every call shares the array and rewrites it (the tables, and the error block is cleared).
 *    Calls that overlap on the GPU race, so issue them on one stream or one after another.
 *  - The call synchronises stream and returns BS_E_CORRUPT if a chunk fails its end check.
 *  - Tables larger than 64 KiB give BS_E_SIZE. No valid container has such a tensor: 64 KiB
 *    is the JOINT table at nj = 13; the largest RANS tables (the s-table at ns = 12 plus 16
 *    fraction rows at nh = 5) take 34 KiB.
 *  - It calls no cudaMalloc, cudaFree or other allocating routine.
 */
bs_status bs_decode_tensor_noalloc(const void* h_container, size_t container_bytes, const void* d_container,
                                   int32_t idx, void* d_out, size_t out_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * Encoder on the device. It produces the canonical container (header, directory, names, then
 * each tensor's model, chunk table and chunks), byte-identical to any other encoder that
 * follows the container's integer rules (quantiser, routes, pad word, STORED fallback). The card's
 * compressor ("bigsmall compress" on the "Gemma 2 9B Instruct -- Lossless Compressed"
 * card, "Want to compress your own model?") is the user-facing counterpart.
 *
 *   1. bs_encoder_create  describes the tensors (device pointers to the originals)
 *   2. bs_encoder_run     histograms, models and a counting pass on the device; returns
 *                         the exact container size
 *   3. bs_encoder_emit    writes the container into caller device memory (and, if asked,
 *                         a host copy)
 *   4. bs_encoder_destroy
 * The originals must stay unchanged on the device from run to emit. All device memory
 * belongs to the caller: the originals, the scratch buffer (bs_encoder_scratch_bytes) and
 * the container.
 * ------------------------------------------------------------------------------------ */
typedef struct bs_encoder_t bs_encoder_t;

typedef struct {
    uint32_t kind;        /* 0: BF16 words (the encoder picks RANS or STORED); 2: RAW bytes */
    uint32_t ndim;
    uint64_t shape[8];
    uint64_t n_elems;     /* words (kind 0) or bytes (kind 2); must equal the shape product */
    const void* d_data;   /* device; 16-byte aligned for kind 0 */
    const char* name;     /* copied at create time */
    uint32_t name_bytes;
    uint32_t reserved;
} bs_enc_item;

typedef struct {
    uint32_t log2_chunk;  /* 8..24, default 16 */
    uint32_t ns;          /* 1..12, default 11 */
    uint32_t nh;          /* 3..5 with ns + nh <= 16, default 5 */
    uint32_t max_routes;  /* 0..15, default 15 */
    uint32_t force_rans;  /* 1: never fall back to STORED (tests only) */
    uint32_t model;       /* 0: factored RANS model (ns, nh, routes); 1: JOINT (one table over (s, h)) */
    uint32_t nj;          /* JOINT precision, 8..13, default 13 */
} bs_enc_params;

bs_status bs_encoder_create(const bs_enc_item* items, int32_t n, const bs_enc_params* params, bs_encoder_t** out);
/* Device scratch for bs_encoder_run / bs_encoder_emit (histograms, tables, chunk sizes). */
bs_status bs_encoder_scratch_bytes(const bs_encoder_t* enc, size_t* bytes);
/* Synchronises stream. *container_bytes receives the size bs_encoder_emit will write. */
bs_status bs_encoder_run(bs_encoder_t* enc, void* d_scratch, size_t scratch_bytes, void* stream,
                         size_t* container_bytes);
/* d_container: container_bytes of device memory, 16-byte aligned. h_container: NULL, or
 * a host buffer of container_bytes that receives a copy. Synchronises stream. */
bs_status bs_encoder_emit(bs_encoder_t* enc, void* d_scratch, void* d_container, size_t container_bytes,
                          void* h_container, void* stream);
void bs_encoder_destroy(bs_encoder_t* enc);

/* ------------------------------------------------------------------------------------
 * Layer streaming: decode groups of tensors on demand from a container in HOST memory
 * into a bounded device cache, with least-recently-used eviction. This is the device
 * counterpart of the low-VRAM streaming loader on the "Gemma 2 9B Instruct -- Lossless
 * Compressed" card (section "Low-VRAM streaming"): layers are decompressed as they are
 * needed, under a cap on device memory (the card's lru_max_vram_gb). The card gives only
 * that API, so the policy and the memory layout below are this library's.
 *
 * group_of_tensor[k] is the group of tensor k (directory order). Group numbers run
 * 0..G-1 and each is used at least once; a group is typically one layer.
 * d_arena is the whole device budget, owned by the caller (256-byte aligned). It holds:
 *   - two staging slots, each the size of the largest group's compressed byte range;
 *   - then the cache of decoded groups.
 * Eviction is least-recently-used among unpinned groups. A prefetched group is kept until it
 * has been acquired once, unless nothing else can make room.
 * Loading a group runs on the stream given to prefetch or acquire, in three steps:
 *   1. one cudaMemcpyAsync host-to-device of the group's compressed bytes into a slot;
 *   2. the decode kernels (the same as bs_decode_batch) into a cache block;
 *   3. events that order the later reuse of the slot and of the block.
 * No call blocks the host, except create (which uploads the tables) and check.
 * For the copies to overlap other work, h_container should be page-locked.
 * h_container must stay valid and unchanged until bs_streamer_destroy.
 * Device memory is never allocated. The library's host memory is freed by destroy.
 * The object is internally locked: calls from several host threads are serialised.
 * After a BS_E_CUDA from prefetch or acquire the cache may have lost the block being loaded
 * (the block is never reused while work may still write into it); destroy and recreate.
 * ------------------------------------------------------------------------------------ */
typedef struct bs_streamer_t bs_streamer_t;

typedef struct {
    uint64_t loads;            /* groups staged and decoded */
    uint64_t hits;             /* acquires that found their group resident */
    uint64_t evictions;        /* groups dropped from the cache to make room */
    uint64_t h2d_bytes;        /* compressed bytes copied host-to-device */
    uint64_t decoded_bytes;    /* bytes of decoded cache blocks written */
    uint64_t resident_groups;  /* groups in the cache now */
    uint64_t cache_bytes;      /* size of the cache part of the arena */
    uint64_t cache_bytes_used; /* bytes of it held by resident groups now */
    uint64_t stage_bytes;      /* size of one staging slot */
} bs_streamer_stats_t;

/* Device workspace bytes (decode tables and error block); 0 if the container fails validation. */
size_t bs_streamer_workspace_bytes(const void* h_container, size_t container_bytes);
/* The smallest arena for this grouping: two staging slots plus the largest decoded group.
 * 0 if the container fails validation or the grouping is invalid. */
size_t bs_streamer_min_arena_bytes(const void* h_container, size_t container_bytes, const int32_t* group_of_tensor);
/* Validate the container (as bs_plan does) and upload the decode tables into d_workspace on
 * stream, then synchronise it. Returns:
 *   BS_E_SIZE when the workspace or the arena is too small;
 *   BS_E_ARG for a bad grouping;
 *   BS_E_UNSUPPORTED off sm_100.
 * The streamer is bound to the current device. */
bs_status bs_streamer_create(const void* h_container, size_t container_bytes, const int32_t* group_of_tensor,
                             void* d_workspace, size_t workspace_bytes, void* d_arena, size_t arena_bytes,
                             void* stream, bs_streamer_t** out);
bs_status bs_streamer_group_count(const bs_streamer_t* s, int32_t* n);
/* As bs_tensor_info_get; the name stays valid until bs_streamer_destroy. */
bs_status bs_streamer_tensor_info_get(const bs_streamer_t* s, int32_t idx, bs_tensor_info* info);
/* Queue the load of a group that is not resident. Returns BS_OK at once if it is resident.
 * Returns BS_E_SIZE when the groups now acquired leave no room for it. */
bs_status bs_streamer_prefetch(bs_streamer_t* s, int32_t group, void* stream);
/* Make the group resident (loading it on `stream` if needed) and pin it.
 * d_ptrs[0..n_ptrs) receives the device address of each of its tensors, in ascending
 * tensor index. RANS/STORED tensors are BF16 words, RAW tensors are bytes, and every
 * address is 256-byte aligned. n_ptrs must equal the group's tensor count (else BS_E_SIZE).
 * Work queued on `stream` after this call sees the decoded data, including a load started
 * on another stream by prefetch. Every acquire needs a matching release. */
bs_status bs_streamer_acquire(bs_streamer_t* s, int32_t group, void** d_ptrs, int32_t n_ptrs, void* stream);
/* Unpin after the work queued on `stream` so far. The group may then be evicted, and its
 * memory is reused only after that work. */
bs_status bs_streamer_release(bs_streamer_t* s, int32_t group, void* stream);
bs_status bs_streamer_get_stats(bs_streamer_t* s, bs_streamer_stats_t* out);
/* As bs_check, for the streamer's error word: synchronises stream. */
bs_status bs_streamer_check(bs_streamer_t* s, void* stream, int64_t* first_bad);
/* Frees host state only. It does not synchronise: finish the streams before freeing the arena. */
void bs_streamer_destroy(bs_streamer_t* s);

/* ------------------------------------------------------------------------------------
 * Fixed-width lane layout ("FW layout"): a runtime form of one BF16
 * tensor whose decode is a few bitwise operations per weight. The "Qwen3.8-27B-BF16-NVLC-
 * Lossless" card says its GPU runtime derives fixed-width, lane-oriented streams from the
 * rANS files once at initialisation (its Fixed7/Compact11 runtime, about 11.36 bits per
 * weight resident). The card gives no layout; this one is this library's:
 *   - a 4-bit code per weight for the tensor's 16 most frequent sign+exponent symbols;
 *   - the 7-bit fraction in two planes;
 *   - an exception list of (position, word) for the other symbols.
 * Tiles of 256 weights: lane j of a warp owns 8 consecutive weights. The size is 11.125
 * bits per weight plus 24 bits per escape, about 11.4 on Gaussian-shaped weights.
 *
 * Building one (on the device, from BF16 words that stay unchanged between the calls):
 *   1. bs_fw_measure: statistics, code table and escape counts into caller scratch;
 *      synchronises the stream and returns the layout's size in info->total_bytes;
 *   2. bs_fw_write: writes the layout into caller device memory; synchronises the stream.
 * Decoding: bs_fw_decode, enqueued on the stream without a sync. All device memory belongs
 * to the caller. The library allocates none.
 * ------------------------------------------------------------------------------------ */
typedef struct {
    uint64_t n_elems;     /* weights */
    uint64_t n_tiles;     /* ceil(n_elems / 256) */
    uint64_t n_exc;       /* escaped weights, below 2^32 */
    uint64_t total_bytes; /* size of the layout in bytes (a multiple of 16) */
    uint16_t table[16];   /* the sign+exponent symbol of each code */
} bs_fw_info;

/* Device scratch bytes of bs_fw_measure / bs_fw_write for n_elems weights (0 if n_elems > 2^40). */
size_t bs_fw_scratch_bytes(uint64_t n_elems);
/* d_in: n_elems BF16 words on the device, 16-byte aligned. d_scratch: 256-byte aligned,
 * at least bs_fw_scratch_bytes(n_elems). Synchronises stream and fills *info.
 * BS_E_SIZE if the scratch is short, n_elems > 2^40, or 2^32 or more weights would escape.
 * BS_E_UNSUPPORTED off sm_100. */
bs_status bs_fw_measure(const void* d_in, uint64_t n_elems, void* d_scratch, size_t scratch_bytes, void* stream,
                        bs_fw_info* info);
/* Writes the layout described by *info (from bs_fw_measure on the same d_in and d_scratch)
 * into d_fw: fw_bytes == info->total_bytes bytes of device memory, 16-byte aligned.
 * Synchronises stream. BS_E_CORRUPT if the input changed since bs_fw_measure. */
bs_status bs_fw_write(const void* d_in, uint64_t n_elems, void* d_scratch, size_t scratch_bytes,
                      const bs_fw_info* info, void* d_fw, size_t fw_bytes, void* stream);
/* Validates a host copy of a layout's first 96 bytes (header and code table) against the
 * layout's size fw_bytes, and fills *info. BS_E_FORMAT or BS_E_VERSION on a bad header. */
bs_status bs_fw_parse(const void* h_head, size_t head_bytes, size_t fw_bytes, bs_fw_info* info);
/* Decodes n layouts in as few launches as possible (up to 480 layouts per launch).
 *   d_fw[k]: layout k on the device, 16-byte aligned, infos[k] its header (from
 *            bs_fw_measure or bs_fw_parse);
 *   d_out[k]: infos[k].n_elems words, 16-byte aligned, out_bytes[k] == 2 * n_elems;
 *   d_err: a device word the caller zeroes before and reads after. An exception list that
 *          fails its checks sets bit 0: tile_exc not ascending or past n_exc within a group of
 *          4 tiles (the group's exceptions are then skipped), or a position past the tensor
 *          (that exception is skipped). Nothing is written outside d_out[k].
 * Enqueued on stream; returns BS_E_ARG / BS_E_SIZE for bad arguments before any launch. */
bs_status bs_fw_decode(int32_t n, const void* const* d_fw, const bs_fw_info* infos, void* const* d_out,
                       const size_t* out_bytes, uint32_t* d_err, void* stream);

/* y = W x with W in the FW layout, decoded in registers on its way to the multiply: no dense
 * copy of W is written. This is the operand path of the NVLC card's runtime (compressed
 * weights resident, no persistent decoded-weight cache). For batch 1..8 the product is bound
 * by the bytes of W, so it runs on the CUDA cores with fp32 accumulation.
 *   d_fw, info: W's layout, rows x cols row-major (rows * cols == info.n_elems), with cols
 *               a multiple of 256 (each row is whole tiles); 16-byte aligned;
 *   d_x:        BF16 [batch][cols], 16-byte aligned;
 *   d_y:        FP32 [batch][rows]; each entry is written once (no accumulation into it).
 * Summation order is fixed, so results are deterministic. Escaped weights enter as the
 * decoded placeholder plus a correction (w_true - w_placeholder) * x. */
typedef struct {
    const void* d_fw;
    bs_fw_info info;
    uint32_t rows, cols;
    const void* d_x;
    float* d_y;
} bs_fw_gemv_item;
/* Computes every item's product, up to 384 items per launch; batch is 1..8 for all items.
 * d_err as for bs_fw_decode. Enqueued on stream.
 * Each launch may be scheduled while the kernel before it on the stream is finishing
 * (programmatic dependent launch): its CTAs take the SMs that kernel leaves. Without flags it
 * reads and writes no global memory before that kernel has completed, so stream order holds
 * as for any launch.
 * flags: 0, or BS_FW_LAYOUTS_RESIDENT: the caller states that no work still in flight on the
 * stream writes any item's layout (d_fw), as for weights written once and kept resident. The
 * kernel then starts copying the layouts as soon as it is scheduled; it still waits for the
 * preceding kernel to complete before it reads x or writes y or d_err. Other bits: BS_E_ARG. */
#define BS_FW_LAYOUTS_RESIDENT 1u
bs_status bs_fw_gemv(int32_t n, const bs_fw_gemv_item* items, uint32_t batch, uint32_t flags, uint32_t* d_err,
                     void* stream);

/* Y = X W^T for a batch of tokens on the tensor cores, W in the FW layout: the same products as
 * bs_fw_gemv (the same items, Y[b][r] = sum_k W[r][k] X[b][k]) for batches too large for the
 * CUDA cores. Source: the NVLC card's runtime keeps the compressed weights resident and no
 * decoded-weight cache (its runtime accounting and DGX Spark tables); the kernel is this
 * library's. W is decoded in blocks of 128 rows, 128 columns of K at a time, into shared
 * memory in the tensor cores' operand layout and multiplied with up to 64 tokens
 * (tcgen05.mma, BF16 operands, FP32 accumulation in tensor memory); larger batches decode
 * each row block once per 64 tokens.
 *   rows must be a multiple of 128 and cols of 256 (else BS_E_ARG); batch is 1..2^20; a matrix
 *   of 2^32 / 128 tiles or more gives BS_E_SIZE.
 *   The work (row blocks x K tiles x token blocks) is shared evenly by one wave of CTAs, so a
 *   row block's K range can be split between CTAs. Every item's Y is zeroed first (on stream)
 *   and split row blocks add their parts with atomic FP32 adds; a part sum over two CTAs does
 *   not depend on their order, but one over three or more (small launches) can differ in its
 *   last bits from run to run.
 *   d_err: as for bs_fw_decode; bit 1 means that a wait inside the kernel ran out (the
 *          outputs of that CTA are then not written).
 * The FP32 sums follow the tensor cores' order, so they may differ from bs_fw_gemv's in the
 * last bits. Enqueued on stream. */
bs_status bs_fw_gemm(int32_t n, const bs_fw_gemv_item* items, uint32_t batch, uint32_t* d_err, void* stream);

/* Diagnostics (this library's design). */
const char* bs_status_str(bs_status s);
int bs_last_cuda_error(void); /* the cudaError_t behind the last BS_E_CUDA on this thread */
/* Kernel launches libbs has made in this process (all threads); a diagnostic counter. */
uint64_t bs_launch_counter(void);

#ifdef __cplusplus
}
#endif
#endif /* BS_H */
