/*
 * fworacle.c -- the oracle for the fixed-width lane layout: a plain, slow,
 * CPU-only encoder and decoder. It is TEST INFRASTRUCTURE. Only the tests, the smoke
 * check and the CPU-baseline leg of bench.py may load it. The GPU library never calls it,
 * and it shares no source with the GPU library.
 *
 * What it computes: the fixed-width, lane-oriented runtime form that the
 * "Qwen3.8-27B-BF16-NVLC-Lossless" card says its GPU runtime derives from the rANS files at
 * initialisation (its Fixed7/Compact11 runtime; the runtime accounting table gives the
 * resident codes plus metadata at about 11.36 bits per weight). The card gives no layout,
 * so the one here is this project's, and each function states the part it follows: a
 * 16-entry code table, planes A (4-bit codes), B (low nibbles) and C (top fraction bits) per
 * 256-weight tile, and an exception list.
 *
 * Pins (tests/test_fw_oracle.py):
 *   - two hand-derived layouts (tests/golden/lane_*.hex);
 *   - a round trip on every 16-bit pattern;
 *   - the size formula checked against a count of escapes done in the test;
 *   - the code table checked against a sort done in the test;
 *   - rejection of each malformed field.
 *
 * Style: one weight at a time, and every bit field is set or read one bit at a time.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Status codes; the same numbers as bsoracle.c. */
enum {
    LO_OK = 0,
    LO_E_ARG = 1,
    LO_E_FORMAT = 2,
    LO_E_VERSION = 3,
    LO_E_SIZE = 4,
    LO_E_CORRUPT = 6,
    LO_E_NOMEM = 7
};

#define LANE_TILE 256u
#define LANE_HEADER 64u
#define LANE_SYMBOLS 512u

static const uint8_t kLaneMagic[8] = {'B', 'F', '1', '6', 'L', 'A', 'N', 'E'};

typedef struct {
    uint64_t n_elems, n_tiles, n_exc, total_bytes;
    uint16_t table[16];
} bso_fw_info;

static uint64_t up16(uint64_t v) { return (v + 15u) & ~(uint64_t)15u; }
static uint64_t get_le(const uint8_t* p, uint32_t bytes) {
    uint64_t v = 0;
    for (uint32_t k = 0; k < bytes; ++k) v |= (uint64_t)p[k] << (8u * k);
    return v;
}
static void put_le(uint8_t* p, uint32_t bytes, uint64_t v) {
    for (uint32_t k = 0; k < bytes; ++k) p[k] = (uint8_t)(v >> (8u * k));
}

/* A bit field of `width` bits starting at bit `bit` of a little-endian byte array
 * (bit b is bit b % 8 of byte b / 8). The layout's u32 planes are little-endian, so
 * bit k of lane j's word is bit 32j + k of the plane's bytes. */
static void set_bits(uint8_t* base, uint64_t bit, uint32_t width, uint32_t value) {
    for (uint32_t b = 0; b < width; ++b)
        if ((value >> b) & 1u) base[(bit + b) >> 3] |= (uint8_t)(1u << ((bit + b) & 7u));
}
static uint32_t get_bits(const uint8_t* base, uint64_t bit, uint32_t width) {
    uint32_t v = 0;
    for (uint32_t b = 0; b < width; ++b) v |= (uint32_t)((base[(bit + b) >> 3] >> ((bit + b) & 7u)) & 1u) << b;
    return v;
}

/* Section 10, byte layout: the section offsets of a layout with n_tiles tiles and n_exc
 * escapes. */
typedef struct {
    uint64_t a, b, c, tile_exc, exc_pos, exc_word, total;
} lane_offsets;

static lane_offsets offsets_of(uint64_t n_tiles, uint64_t n_exc) {
    lane_offsets o;
    o.a = LANE_HEADER + 32u;
    o.b = o.a + 128u * n_tiles;
    o.c = o.b + 128u * n_tiles;
    o.tile_exc = o.c + 96u * n_tiles;
    o.exc_pos = o.tile_exc + up16(4u * (n_tiles + 1u));
    o.exc_word = o.exc_pos + up16(n_exc);
    o.total = o.exc_word + up16(2u * n_exc);
    return o;
}

/* Section 10, byte layout: the size of the layout of n_elems weights with n_exc escapes. */
uint64_t bso_fw_bytes(uint64_t n_elems, uint64_t n_exc) {
    return offsets_of((n_elems + LANE_TILE - 1u) / LANE_TILE, n_exc).total;
}

/* Section 10, code table: the present symbols by decreasing count, ties to the lower s, at
 * most 16; unused entries 0. Found by picking the largest remaining count 16 times. */
int bso_fw_table(const uint16_t* w, uint64_t n, uint16_t* table, uint32_t* n_codes) {
    if ((!w && n) || !table) return LO_E_ARG;
    uint64_t* count = (uint64_t*)calloc(LANE_SYMBOLS, sizeof(uint64_t));
    uint8_t* taken = (uint8_t*)calloc(LANE_SYMBOLS, 1);
    if (!count || !taken) {
        free(count);
        free(taken);
        return LO_E_NOMEM;
    }
    for (uint64_t i = 0; i < n; ++i) count[w[i] >> 7]++;
    uint32_t k = 0;
    for (; k < 16u; ++k) {
        int best = -1;
        for (uint32_t s = 0; s < LANE_SYMBOLS; ++s) /* ascending s, strict >: ties keep the lower s */
            if (!taken[s] && count[s] > 0 && (best < 0 || count[s] > count[best])) best = (int)s;
        if (best < 0) break;
        table[k] = (uint16_t)best;
        taken[best] = 1;
    }
    for (uint32_t r = k; r < 16u; ++r) table[r] = 0;
    if (n_codes) *n_codes = k;
    free(count);
    free(taken);
    return LO_OK;
}

/* Section 10: encode n weights. With out == NULL only *out_bytes is set (a size query).
 * Otherwise out must hold cap >= *out_bytes bytes, else LO_E_SIZE. */
int bso_fw_encode(const uint16_t* w, uint64_t n, uint8_t* out, uint64_t cap, uint64_t* out_bytes) {
    if ((!w && n) || !out_bytes) return LO_E_ARG;
    uint16_t table[16];
    uint32_t n_codes = 0;
    int st = bso_fw_table(w, n, table, &n_codes);
    if (st) return st;
    int code_of[LANE_SYMBOLS];
    for (uint32_t s = 0; s < LANE_SYMBOLS; ++s) code_of[s] = -1;
    for (uint32_t k = 0; k < n_codes; ++k) code_of[table[k]] = (int)k;

    uint64_t n_exc = 0;
    for (uint64_t i = 0; i < n; ++i)
        if (code_of[w[i] >> 7] < 0) n_exc++;
    if (n_exc >= (1ull << 32)) return LO_E_SIZE;
    const uint64_t n_tiles = (n + LANE_TILE - 1u) / LANE_TILE;
    const lane_offsets o = offsets_of(n_tiles, n_exc);
    *out_bytes = o.total;
    if (!out) return LO_OK;
    if (cap < o.total) return LO_E_SIZE;
    memset(out, 0, o.total);

    memcpy(out, kLaneMagic, 8);
    put_le(out + 8, 4, 1);
    put_le(out + 12, 4, LANE_HEADER);
    put_le(out + 16, 8, n);
    put_le(out + 24, 8, n_tiles);
    put_le(out + 32, 8, n_exc);
    put_le(out + 40, 8, o.total);
    for (uint32_t k = 0; k < 16u; ++k) put_le(out + LANE_HEADER + 2u * k, 2, table[k]);

    uint64_t e = 0; /* escapes so far */
    for (uint64_t i = 0; i < n_tiles * LANE_TILE; ++i) {
        const uint64_t T = i / LANE_TILE;
        const uint32_t pos = (uint32_t)(i % LANE_TILE), j = pos / 8u, t = pos % 8u;
        if (pos == 0) put_le(out + o.tile_exc + 4u * T, 4, e);
        uint32_t code = 0, f = 0;                     /* padding: code 0, fraction 0 */
        if (i < n) {
            const uint32_t s = w[i] >> 7;
            f = w[i] & 0x7Fu;
            if (code_of[s] >= 0) {
                code = (uint32_t)code_of[s];
            } else {                                  /* an escape: code 0 and one exception */
                out[o.exc_pos + e] = (uint8_t)pos;
                put_le(out + o.exc_word + 2u * e, 2, w[i]);
                e++;
            }
        }
        const uint32_t u = f & 15u, h = f >> 4;
        set_bits(out + o.a + 128u * T, 32u * j + 4u * t, 4, code);
        set_bits(out + o.b + 128u * T, 32u * j + 4u * (t >> 1) + 16u * (t & 1u), 4, u);
        set_bits(out + o.c + 96u * T, 24u * j + 3u * (t >> 1) + 12u * (t & 1u), 3, h);
    }
    put_le(out + o.tile_exc + 4u * n_tiles, 4, e);
    return LO_OK;
}

/* Section 10, validation of the header and the code table against the buffer size. */
int bso_fw_parse(const uint8_t* b, uint64_t len, bso_fw_info* info) {
    if (!b || !info) return LO_E_ARG;
    if (len < LANE_HEADER + 32u) return LO_E_FORMAT;
    if (memcmp(b, kLaneMagic, 8) != 0) return LO_E_FORMAT;
    if (get_le(b + 8, 4) != 1u) return LO_E_VERSION;
    if (get_le(b + 12, 4) != LANE_HEADER) return LO_E_FORMAT;
    const uint64_t n = get_le(b + 16, 8), nt = get_le(b + 24, 8), ne = get_le(b + 32, 8), tot = get_le(b + 40, 8);
    if (n > (1ull << 40)) return LO_E_FORMAT;
    if (nt != (n + LANE_TILE - 1u) / LANE_TILE) return LO_E_FORMAT;
    if (ne >= (1ull << 32) || ne > n) return LO_E_FORMAT;
    if (tot != offsets_of(nt, ne).total || tot != len) return LO_E_FORMAT;
    for (uint32_t k = 48; k < 64; ++k)
        if (b[k]) return LO_E_FORMAT;
    for (uint32_t k = 0; k < 16u; ++k) {
        info->table[k] = (uint16_t)get_le(b + LANE_HEADER + 2u * k, 2);
        if (info->table[k] >= LANE_SYMBOLS) return LO_E_FORMAT;
    }
    info->n_elems = n;
    info->n_tiles = nt;
    info->n_exc = ne;
    info->total_bytes = tot;
    return LO_OK;
}

/* Section 10, decoding: every weight from its code, low nibble and top bits, then each
 * listed exception replaces its weight. The exception lists are checked in full: tile_exc
 * starts at 0, never decreases and ends at n_exc, and the positions of a tile ascend and
 * lie inside the tensor. Anything else is LO_E_CORRUPT. */
int bso_fw_decode(const uint8_t* b, uint64_t len, uint16_t* out, uint64_t n_out) {
    bso_fw_info info;
    int st = bso_fw_parse(b, len, &info);
    if (st) return st;
    if (n_out != info.n_elems || (!out && n_out)) return LO_E_SIZE;
    const lane_offsets o = offsets_of(info.n_tiles, info.n_exc);
    for (uint64_t i = 0; i < info.n_elems; ++i) {
        const uint64_t T = i / LANE_TILE;
        const uint32_t pos = (uint32_t)(i % LANE_TILE), j = pos / 8u, t = pos % 8u;
        const uint32_t code = get_bits(b + o.a + 128u * T, 32u * j + 4u * t, 4);
        const uint32_t u = get_bits(b + o.b + 128u * T, 32u * j + 4u * (t >> 1) + 16u * (t & 1u), 4);
        const uint32_t h = get_bits(b + o.c + 96u * T, 24u * j + 3u * (t >> 1) + 12u * (t & 1u), 3);
        out[i] = (uint16_t)((info.table[code] << 7) | (h << 4) | u);
    }
    if (get_le(b + o.tile_exc, 4) != 0) return LO_E_CORRUPT;
    for (uint64_t T = 0; T < info.n_tiles; ++T) {
        const uint64_t e0 = get_le(b + o.tile_exc + 4u * T, 4), e1 = get_le(b + o.tile_exc + 4u * (T + 1u), 4);
        if (e1 < e0 || e1 > info.n_exc) return LO_E_CORRUPT;
        for (uint64_t k = e0; k < e1; ++k) {
            const uint32_t pos = b[o.exc_pos + k];
            if (k > e0 && pos <= b[o.exc_pos + k - 1u]) return LO_E_CORRUPT;
            if (T * LANE_TILE + pos >= info.n_elems) return LO_E_CORRUPT;
            out[T * LANE_TILE + pos] = (uint16_t)get_le(b + o.exc_word + 2u * k, 2);
        }
    }
    if (get_le(b + o.tile_exc + 4u * info.n_tiles, 4) != info.n_exc) return LO_E_CORRUPT;
    return LO_OK;
}
