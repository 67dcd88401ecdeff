/*
 * bsoracle.c -- the oracle: a plain, slow, CPU-only encoder and decoder for the
 * BF16RANS container, version 2. It is TEST INFRASTRUCTURE. Only the tests, the
 * smoke check and the CPU-baseline leg of bench.py may load it. The GPU library
 * never calls it, and it shares no source with the GPU library.
 *
 * What it computes follows the "Qwen3.8-27B-BF16-NVLC-Lossless" model card, in the
 * paragraph after its accounting table:
 *   - each BF16 word is split into its exact sign:1 | exponent:8 | fraction:7 fields;
 *   - the joint sign+exponent symbol is coded with a per-tensor rANS model;
 *   - the decoded symbol selects the distribution for the 7-bit fraction (here: a
 *     table over the fraction's top three bits, with the low four bits verbatim);
 *   - the fields are recombined bitwise;
 *   - a residual stream keeps non-BF16 bytes verbatim (RAW kind here).
 * The card gives no byte layout, rANS parameters, interleaving or quantiser. Those are
 * this project's container (BF16RANS version 2), and each function states the rule it
 * follows: 32-bit states in [2^16, 2^32), 16-bit renormalisation words, 32 lanes per
 * chunk under the octet map, words interleaved in (step, lane) order, the integer
 * quantiser and route rule, and the byte layout.
 *
 * The JOINT kind codes the pair (s, h) with one table of 2^nj slots instead of the
 * factored s-model and routes; model_t.joint selects it.
 *
 * Pins (tests/test_oracle_*.py):
 *   - round trip on every 16-bit pattern;
 *   - brute force over tiny alphabets;
 *   - hand-derived containers (the .hex files under tests/golden, each with its derivation);
 *   - Gibbs' inequality and a stated overhead bound against the empirical entropy;
 *   - closed forms of the quantiser.
 *
 * Style: the code is deliberately unoptimised. There is one loop per definition and
 * one symbol at a time. Symbol lookup expands each table into a slot array.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Status codes returned by every exported function. */
enum {
    BSO_OK = 0,
    BSO_E_ARG = 1,
    BSO_E_FORMAT = 2,
    BSO_E_VERSION = 3,
    BSO_E_SIZE = 4,
    BSO_E_CORRUPT = 6,
    BSO_E_NOMEM = 7
};

enum { KIND_RANS = 0, KIND_STORED = 1, KIND_RAW = 2, KIND_JOINT = 3 };
#define JOINT_PAIRS 4096 /* j = (s << 3) | h */

/* RANS and JOINT tensors carry chunks of interleaved rANS lanes. */
static int is_coded(uint32_t kind) { return kind == KIND_RANS || kind == KIND_JOINT; }

#define LANES 32
#define HEADER_BYTES 64
#define DIR_ENTRY_BYTES 144
#define STATE_L 65536u /* L = 2^16: the encoder's start state and the decoder's end state */
#define FORMAT_VERSION 2

/* ------------------------------------------------------------------ */
/* little-endian helpers                                              */
/* ------------------------------------------------------------------ */
static uint64_t rd_u64(const uint8_t* p) {
    uint64_t v = 0;
    for (int k = 7; k >= 0; k--) v = (v << 8) | p[k];
    return v;
}
static uint32_t rd_u32(const uint8_t* p) {
    return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}
static uint16_t rd_u16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static void wr_u64(uint8_t* p, uint64_t v) {
    for (int k = 0; k < 8; k++) { p[k] = (uint8_t)(v & 0xFF); v >>= 8; }
}
static void wr_u32(uint8_t* p, uint32_t v) {
    for (int k = 0; k < 4; k++) { p[k] = (uint8_t)(v & 0xFF); v >>= 8; }
}
static void wr_u16(uint8_t* p, uint16_t v) { p[0] = (uint8_t)(v & 0xFF); p[1] = (uint8_t)(v >> 8); }
static uint64_t align16(uint64_t v) { return (v + 15u) & ~(uint64_t)15u; }

/* ------------------------------------------------------------------ */
/* Checksum: sum of splitmix64 outputs; mix64 = the output for state v */
/* ------------------------------------------------------------------ */
uint64_t bso_mix64(uint64_t v) {
    uint64_t z = v + 0x9E3779B97F4A7C15ULL;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* kind RAW: bytes, position shift 8; otherwise 16-bit words, shift 16 */
uint64_t bso_checksum(const void* data, uint64_t n, uint32_t kind) {
    uint64_t sum = 0;
    if (kind == 2) {
        const uint8_t* b = (const uint8_t*)data;
        for (uint64_t i = 0; i < n; i++) sum += bso_mix64((i << 8) | b[i]);
    } else {
        const uint16_t* w = (const uint16_t*)data;
        for (uint64_t i = 0; i < n; i++) sum += bso_mix64((i << 16) | w[i]);
    }
    return sum;
}

/* ------------------------------------------------------------------ */
/* Quantiser: proportional with a floor of 1, fixed one unit at a time */
/* ------------------------------------------------------------------ */
/* Is a/b > c/d ?  (all non-negative; b, d > 0) */
static int ratio_gt(uint64_t a, uint64_t b, uint64_t c, uint64_t d) {
    return (unsigned __int128)a * d > (unsigned __int128)c * b;
}

/* q[k] = quantised frequency of symbol k so that sum(q) = M; present symbols get >= 1.
 * Returns BSO_E_ARG if more symbols are present than M slots. */
int bso_quantise(const uint64_t* c, uint32_t K, uint32_t M, uint32_t* q) {
    uint64_t n = 0, present = 0;
    for (uint32_t k = 0; k < K; k++) { n += c[k]; if (c[k]) present++; }
    if (n == 0 || present > M) return BSO_E_ARG;
    uint64_t sum = 0;
    for (uint32_t k = 0; k < K; k++) {
        if (c[k] == 0) { q[k] = 0; continue; }
        unsigned __int128 num = (unsigned __int128)2 * c[k] * M + n;
        uint64_t v = (uint64_t)(num / ((unsigned __int128)2 * n));
        q[k] = (uint32_t)(v < 1 ? 1 : v);
        sum += q[k];
    }
    while (sum < M) { /* add one where c/(2q+1) is largest */
        int best = -1;
        for (uint32_t k = 0; k < K; k++) {
            if (!c[k]) continue;
            if (best < 0 || ratio_gt(c[k], 2ull * q[k] + 1, c[best], 2ull * q[best] + 1)) best = (int)k;
        }
        q[best] += 1;
        sum += 1;
    }
    while (sum > M) { /* remove one where c/(2q-1) is smallest, among q >= 2 */
        int best = -1;
        for (uint32_t k = 0; k < K; k++) {
            if (!c[k] || q[k] < 2) continue;
            if (best < 0 || ratio_gt(c[best], 2ull * q[best] - 1, c[k], 2ull * q[k] - 1)) best = (int)k;
        }
        if (best < 0) return BSO_E_ARG; /* cannot happen when present <= M */
        q[best] -= 1;
        sum -= 1;
    }
    return BSO_OK;
}


/* ------------------------------------------------------------------ */
/* Route choice: Pearson statistic of the top fraction bits            */
/* ------------------------------------------------------------------ */
/* ceh: 256*8 counts of the fraction's top three bits, row e = exponent. Writes
 * route[256] and the ascending exponent list route_e[0..n_routes-1]. */
int bso_choose_routes(const uint64_t* ceh, uint32_t max_routes, uint8_t* route, uint32_t* n_routes_out,
                      uint32_t* route_e) {
    unsigned __int128 num[256]; /* chi2_e * n_e = 8*S_e - n_e^2 */
    uint64_t ne[256];
    int cand[256];
    if (max_routes > 15) return BSO_E_ARG;
    for (int e = 0; e < 256; e++) {
        unsigned __int128 S = 0;
        uint64_t n = 0;
        for (int h = 0; h < 8; h++) {
            uint64_t v = ceh[e * 8 + h];
            n += v;
            S += (unsigned __int128)v * v;
        }
        ne[e] = n;
        num[e] = 8 * S - (unsigned __int128)n * n;
        /* candidate: chi2 > 256  <=>  8 S - n^2 > 256 n */
        cand[e] = (n > 0) && (num[e] > (unsigned __int128)256 * n);
        route[e] = 0xFF;
    }
    /* take candidates by decreasing chi2 (= num/n), ties to lower e */
    int chosen[256] = {0};
    uint32_t taken = 0;
    while (taken < max_routes) {
        int best = -1;
        for (int e = 0; e < 256; e++) {
            if (!cand[e] || chosen[e]) continue;
            if (best < 0) { best = e; continue; }
            /* num[e]/ne[e] > num[best]/ne[best] ? */
            unsigned __int128 lhs = num[e] * ne[best], rhs = num[best] * ne[e];
            if (lhs > rhs) best = e;
        }
        if (best < 0) break;
        chosen[best] = 1;
        taken++;
    }
    uint32_t r = 0;
    for (int e = 0; e < 256; e++)
        if (chosen[e]) { route[e] = (uint8_t)r; route_e[r] = (uint32_t)e; r++; }
    *n_routes_out = r;
    return BSO_OK;
}

/* ------------------------------------------------------------------ */
/* Per-tensor model: s-model, routes and h tables, or the pair table    */
/* ------------------------------------------------------------------ */
typedef struct {
    uint32_t ns, nh, n_routes;
    uint32_t Fs[512], cum_s[512];
    uint8_t route[256];
    uint32_t Fh[16][8], cum_h[16][8]; /* route tables over h; row index = route */
    uint32_t Fu, n_present;           /* UNIFORM frequency = Mh/8 */
    /* decode lookups (slot -> symbol) */
    uint16_t* s_of_slot; /* Ms entries */
    uint8_t* h_of_slot;  /* (n_routes + 1) * Mh entries, last row = UNIFORM */
    /* the joint model (kind JOINT): one table over the pairs j = (s << 3) | h */
    uint32_t joint, nj;
    uint32_t Fj[JOINT_PAIRS], cum_j[JOINT_PAIRS];
    uint16_t* j_of_slot; /* 2^nj entries */
} model_t;

static void model_free(model_t* m) {
    free(m->s_of_slot);
    free(m->h_of_slot);
    free(m->j_of_slot);
    m->s_of_slot = NULL;
    m->h_of_slot = NULL;
    m->j_of_slot = NULL;
}

/* Joint model: cum(j) = Fj[0] + ... + Fj[j-1] and the slot -> pair lookup */
static int joint_build(model_t* m) {
    uint32_t acc = 0;
    for (int j = 0; j < JOINT_PAIRS; j++) { m->cum_j[j] = acc; acc += m->Fj[j]; }
    m->j_of_slot = (uint16_t*)malloc(sizeof(uint16_t) << m->nj);
    if (!m->j_of_slot) return BSO_E_NOMEM;
    for (int j = 0; j < JOINT_PAIRS; j++)
        for (uint32_t k = 0; k < m->Fj[j]; k++) m->j_of_slot[m->cum_j[j] + k] = (uint16_t)j;
    return BSO_OK;
}

static void model_cums(model_t* m) {
    uint32_t acc = 0;
    for (int s = 0; s < 512; s++) { m->cum_s[s] = acc; acc += m->Fs[s]; }
    for (uint32_t r = 0; r < m->n_routes; r++) {
        acc = 0;
        for (int h = 0; h < 8; h++) { m->cum_h[r][h] = acc; acc += m->Fh[r][h]; }
    }
    m->Fu = (1u << m->nh) / 8u;
}

/* frequency and cumulative of top bits h under the table that exponent e selects */
static void frac_model(const model_t* m, uint32_t e, uint32_t h, uint32_t* q, uint32_t* cum) {
    uint8_t r = m->route[e];
    if (r == 0xFF) { *q = m->Fu; *cum = m->Fu * h; }
    else { *q = m->Fh[r][h]; *cum = m->cum_h[r][h]; }
}

static int model_build_lookups(model_t* m) {
    uint32_t Ms = 1u << m->ns, Mh = 1u << m->nh;
    m->s_of_slot = (uint16_t*)malloc(sizeof(uint16_t) * Ms);
    m->h_of_slot = (uint8_t*)malloc((size_t)(m->n_routes + 1) * Mh);
    if (!m->s_of_slot || !m->h_of_slot) return BSO_E_NOMEM;
    for (int s = 0; s < 512; s++)
        for (uint32_t k = 0; k < m->Fs[s]; k++) m->s_of_slot[m->cum_s[s] + k] = (uint16_t)s;
    for (uint32_t r = 0; r <= m->n_routes; r++) {
        uint8_t* row = m->h_of_slot + (size_t)r * Mh;
        for (int h = 0; h < 8; h++) {
            uint32_t q, cum;
            if (r == m->n_routes) { q = m->Fu; cum = m->Fu * (uint32_t)h; }
            else { q = m->Fh[r][h]; cum = m->cum_h[r][h]; }
            for (uint32_t k = 0; k < q; k++) row[cum + k] = (uint8_t)h;
        }
    }
    return BSO_OK;
}

/* ------------------------------------------------------------------ */
/* One lane: encode backwards from L, at most one word per step       */
/* ------------------------------------------------------------------ */
/* Encode the lane's S weights (given in decode order) backwards from x = L. Only the
 * fields s and h go through the state; the nibbles are stored apart.
 * emitted[t] = 1 and word[t] = the word if the lane emitted while encoding step t. */
static uint32_t lane_encode(const model_t* m, const uint16_t* w, uint32_t S, uint8_t* emitted, uint16_t* word) {
    uint32_t x = STATE_L;
    uint32_t P = m->ns + m->nh;
    if (m->joint) { /* the JOINT kind: Q = Fj[j] out of 2^nj */
        for (uint32_t tt = S; tt-- > 0;) {
            uint32_t j = w[tt] >> 4;
            uint64_t Q = m->Fj[j];
            emitted[tt] = 0;
            if ((uint64_t)x >= (Q << (32 - m->nj))) {
                emitted[tt] = 1;
                word[tt] = (uint16_t)(x & 0xFFFFu);
                x >>= 16;
            }
            x = (uint32_t)(((uint64_t)x / Q << m->nj) + m->cum_j[j] + (uint64_t)x % Q);
        }
        return x;
    }
    for (uint32_t tt = S; tt-- > 0;) {
        uint32_t s = w[tt] >> 7, h = (w[tt] >> 4) & 7u, e = s & 0xFF;
        uint32_t qs = m->Fs[s], cs = m->cum_s[s], qh, ch;
        frac_model(m, e, h, &qh, &ch);
        uint64_t Q = (uint64_t)qs * qh;
        emitted[tt] = 0;
        if ((uint64_t)x >= (Q << (32 - P))) { /* renormalise: one word at most */
            emitted[tt] = 1;
            word[tt] = (uint16_t)(x & 0xFFFFu);
            x >>= 16;
        }
        uint64_t k = x % Q;
        x = (uint32_t)(((uint64_t)x / Q << P) + ((cs + k / qh) << m->nh) + ch + k % qh);
    }
    return x;
}

/* ------------------------------------------------------------------ */
/* Single-lane entry points for the brute-force pins                  */
/* ------------------------------------------------------------------ */
/* Tables are given directly: Fs[512] (sum 2^ns), route[256], Fh[n_routes][8]. */
static int model_from_tables(model_t* m, const uint32_t* Fs, uint32_t ns, const uint8_t* route, const uint32_t* Fh,
                             uint32_t n_routes, uint32_t nh) {
    memset(m, 0, sizeof(*m));
    if (ns < 1 || ns > 12 || nh < 3 || nh > 5 || ns + nh > 16 || n_routes > 15) return BSO_E_ARG;
    m->ns = ns; m->nh = nh; m->n_routes = n_routes;
    uint64_t sum = 0;
    for (int s = 0; s < 512; s++) { m->Fs[s] = Fs[s]; sum += Fs[s]; }
    if (sum != (1u << ns)) return BSO_E_ARG;
    for (int e = 0; e < 256; e++) {
        m->route[e] = route[e];
        if (route[e] != 0xFF && route[e] >= n_routes) return BSO_E_ARG;
    }
    for (uint32_t r = 0; r < n_routes; r++) {
        sum = 0;
        for (int h = 0; h < 8; h++) { m->Fh[r][h] = Fh[r * 8 + h]; sum += Fh[r * 8 + h]; }
        if (sum != (1u << nh)) return BSO_E_ARG;
    }
    model_cums(m);
    return BSO_OK;
}

/* Every word must have a nonzero frequency under the tables. */
int bso_lane_encode(const uint32_t* Fs, uint32_t ns, const uint8_t* route, const uint32_t* Fh, uint32_t n_routes,
                    uint32_t nh, const uint16_t* w, uint32_t S, uint32_t* state_out, uint16_t* words_out,
                    uint32_t* tags_out, uint32_t* n_words_out) {
    model_t* m = (model_t*)calloc(1, sizeof(model_t));
    if (!m) return BSO_E_NOMEM;
    int st = model_from_tables(m, Fs, ns, route, Fh, n_routes, nh);
    if (st) { free(m); return st; }
    for (uint32_t t = 0; t < S; t++) {
        uint32_t s = w[t] >> 7, qh, ch;
        frac_model(m, s & 0xFF, (w[t] >> 4) & 7u, &qh, &ch);
        if (m->Fs[s] == 0 || qh == 0) { free(m); return BSO_E_ARG; }
    }
    uint8_t* em = (uint8_t*)malloc(S ? S : 1);
    uint16_t* wd = (uint16_t*)malloc(sizeof(uint16_t) * (S ? S : 1));
    if (!em || !wd) { free(em); free(wd); free(m); return BSO_E_NOMEM; }
    *state_out = lane_encode(m, w, S, em, wd);
    uint32_t k = 0;
    for (uint32_t t = 0; t < S; t++)
        if (em[t]) { words_out[k] = wd[t]; tags_out[k] = t; k++; }
    *n_words_out = k;
    free(em);
    free(wd);
    free(m);
    return BSO_OK;
}

/* Decode S weights of one lane; words are consumed in order, nib[t] is the stored low
 * nibble of weight t. Returns BSO_E_CORRUPT if the end state is not L or the word count
 * does not match. */
int bso_lane_decode(const uint32_t* Fs, uint32_t ns, const uint8_t* route, const uint32_t* Fh, uint32_t n_routes,
                    uint32_t nh, uint32_t state, const uint16_t* words, uint32_t n_words, const uint8_t* nib,
                    uint32_t S, uint16_t* out, uint32_t* final_state) {
    model_t* mp = (model_t*)calloc(1, sizeof(model_t));
    if (!mp) return BSO_E_NOMEM;
    int st = model_from_tables(mp, Fs, ns, route, Fh, n_routes, nh);
    if (st) { free(mp); return st; }
    if ((st = model_build_lookups(mp))) { model_free(mp); free(mp); return st; }
    const model_t* m = mp;
    uint32_t x = state, P = ns + nh;
    uint32_t pos = 0, Mh = 1u << nh;
    int bad = x < STATE_L;
    for (uint32_t t = 0; t < S; t++) {
        uint32_t slot = x & ((1u << P) - 1u);
        uint32_t js = slot >> nh, jh = slot & (Mh - 1u);
        uint32_t s = m->s_of_slot[js];
        uint8_t r = m->route[s & 0xFF];
        uint32_t row = (r == 0xFF) ? m->n_routes : r, qh, ch;
        uint32_t h = m->h_of_slot[(size_t)row * Mh + jh];
        frac_model(m, s & 0xFF, h, &qh, &ch);
        x = m->Fs[s] * qh * (x >> P) + (js - m->cum_s[s]) * qh + (jh - ch);
        if (x < STATE_L) {
            uint32_t wd = 0;
            if (pos < n_words) wd = words[pos]; else bad = 1;
            pos++;
            x = (x << 16) | wd;
        }
        out[t] = (uint16_t)((s << 7) | (h << 4) | (nib[t] & 15u));
    }
    *final_state = x;
    model_free(mp);
    free(mp);
    if (bad || x != STATE_L || pos != n_words) return BSO_E_CORRUPT;
    return BSO_OK;
}

/* The JOINT kind, one lane: the pair table Fj[4096] is given directly (sum 2^nj,
 * 8 <= nj <= 13). Encoding and the tags are as for bso_lane_encode; only the pair
 * j = w >> 4 goes through the state. */
static int joint_model_from_table(model_t* m, const uint32_t* Fj, uint32_t nj) {
    memset(m, 0, sizeof(*m));
    if (nj < 8 || nj > 13) return BSO_E_ARG;
    uint64_t sum = 0;
    for (int j = 0; j < JOINT_PAIRS; j++) { m->Fj[j] = Fj[j]; sum += Fj[j]; }
    if (sum != (1u << nj)) return BSO_E_ARG;
    m->joint = 1;
    m->nj = nj;
    return joint_build(m);
}

int bso_joint_lane_encode(const uint32_t* Fj, uint32_t nj, const uint16_t* w, uint32_t S, uint32_t* state_out,
                          uint16_t* words_out, uint32_t* tags_out, uint32_t* n_words_out) {
    model_t* m = (model_t*)calloc(1, sizeof(model_t));
    if (!m) return BSO_E_NOMEM;
    int st = joint_model_from_table(m, Fj, nj);
    for (uint32_t t = 0; !st && t < S; t++)
        if (m->Fj[w[t] >> 4] == 0) st = BSO_E_ARG;
    uint8_t* em = (uint8_t*)malloc(S ? S : 1);
    uint16_t* wd = (uint16_t*)malloc(sizeof(uint16_t) * (S ? S : 1));
    if (!st && (!em || !wd)) st = BSO_E_NOMEM;
    if (!st) {
        *state_out = lane_encode(m, w, S, em, wd);
        uint32_t k = 0;
        for (uint32_t t = 0; t < S; t++)
            if (em[t]) { words_out[k] = wd[t]; tags_out[k] = t; k++; }
        *n_words_out = k;
    }
    free(em);
    free(wd);
    model_free(m);
    free(m);
    return st;
}

/* Decode S weights of one JOINT lane from `state`, taking words in order; nib[t] is the
 * low nibble of weight t. BSO_E_CORRUPT unless the lane ends at L with every word used. */
int bso_joint_lane_decode(const uint32_t* Fj, uint32_t nj, uint32_t state, const uint16_t* words, uint32_t n_words,
                          const uint8_t* nib, uint32_t S, uint16_t* out, uint32_t* final_state) {
    model_t* m = (model_t*)calloc(1, sizeof(model_t));
    if (!m) return BSO_E_NOMEM;
    int st = joint_model_from_table(m, Fj, nj);
    if (st) { model_free(m); free(m); return st; }
    uint32_t x = state, pos = 0;
    int bad = x < STATE_L;
    for (uint32_t t = 0; t < S; t++) {
        uint32_t slot = x & ((1u << nj) - 1u);
        uint32_t j = m->j_of_slot[slot];
        x = m->Fj[j] * (x >> nj) + (slot - m->cum_j[j]);
        if (x < STATE_L) {
            uint32_t wd = 0;
            if (pos < n_words) wd = words[pos]; else bad = 1;
            pos++;
            x = (x << 16) | wd;
        }
        out[t] = (uint16_t)((j << 4) | (nib[t] & 15u));
    }
    *final_state = x;
    model_free(m);
    free(m);
    if (bad || x != STATE_L || pos != n_words) return BSO_E_CORRUPT;
    return BSO_OK;
}

/* ------------------------------------------------------------------ */
/* Encoder of one BF16 tensor: model, chunks, lanes, payloads          */
/* ------------------------------------------------------------------ */
typedef struct {
    uint8_t* model; /* serialized model, model_bytes long */
    uint64_t model_bytes;
    uint64_t n_chunks;
    uint8_t** chunk; /* each chunk's payload, padded to 16 */
    uint64_t* chunk_bytes;
    uint32_t* chunk_words;
    uint64_t coded_total; /* model + 16*n_chunks + sum chunk bytes */
    uint32_t n_routes;
    uint32_t nib_mode; /* 0 = stored nibble words, 0x10 + c = every low nibble is c */
} rans_blob_t;

static void blob_free(rans_blob_t* b) {
    if (b->chunk)
        for (uint64_t c = 0; c < b->n_chunks; c++) free(b->chunk[c]);
    free(b->chunk);
    free(b->chunk_bytes);
    free(b->chunk_words);
    free(b->model);
    memset(b, 0, sizeof(*b));
}

/* local weight index of (step t, lane j) under the octet map: block t >> 3, lane j, weight t & 7 */
static uint64_t octet_index(uint32_t t, uint32_t j) { return ((uint64_t)(t >> 3) << 8) + 8u * j + (t & 7u); }

/* bit position of the nibble of step t inside its lane's block word: pair (t & 7) >> 1 at bit 4p,
 * the odd step 16 bits higher */
static uint32_t nibble_shift(uint32_t t) { return 4u * ((t & 7u) >> 1) + 16u * (t & 1u); }

static int encode_rans(const uint16_t* w, uint64_t n, uint32_t log2_chunk, uint32_t ns, uint32_t nh,
                       uint32_t max_routes, uint32_t joint, uint32_t nj, rans_blob_t* out) {
    memset(out, 0, sizeof(*out));
    model_t* m = (model_t*)calloc(1, sizeof(model_t));
    uint64_t* cs = (uint64_t*)calloc(512, sizeof(uint64_t));
    uint64_t* ceh = (uint64_t*)calloc(256 * 8, sizeof(uint64_t));
    uint64_t* cj = (uint64_t*)calloc(JOINT_PAIRS, sizeof(uint64_t));
    int st = BSO_E_NOMEM;
    if (!m || !cs || !ceh || !cj) goto done;
    m->ns = ns; m->nh = nh;
    /* counts */
    for (uint64_t i = 0; i < n; i++) {
        uint32_t s = w[i] >> 7;
        cs[s]++;
        ceh[(s & 0xFF) * 8 + ((w[i] >> 4) & 7u)]++;
        cj[w[i] >> 4]++;
    }
    uint16_t pad;
    if (joint) { /* Fj = quantise(pair counts, 2^nj); the pad pair has the largest Fj, lowest j on ties */
        m->joint = 1;
        m->nj = nj;
        if ((st = bso_quantise(cj, JOINT_PAIRS, 1u << nj, m->Fj))) goto done;
        if ((st = joint_build(m))) goto done;
        uint32_t j_pad = 0;
        for (uint32_t j = 1; j < JOINT_PAIRS; j++)
            if (m->Fj[j] > m->Fj[j_pad]) j_pad = j;
        pad = (uint16_t)(j_pad << 4);
        uint32_t n_pairs = 0;
        for (int j = 0; j < JOINT_PAIRS; j++) if (m->Fj[j]) n_pairs++;
        out->model_bytes = 4 + 4ull * n_pairs; /* n_pairs, reserved, (j, Fj) pairs */
        out->model = (uint8_t*)calloc(1, out->model_bytes);
        if (!out->model) { st = BSO_E_NOMEM; goto done; }
        wr_u16(out->model, (uint16_t)n_pairs);
        uint64_t o = 4;
        for (int j = 0; j < JOINT_PAIRS; j++)
            if (m->Fj[j]) { wr_u16(out->model + o, (uint16_t)j); wr_u16(out->model + o + 2, (uint16_t)m->Fj[j]); o += 4; }
        goto chunks;
    }
    /* s-model */
    if ((st = bso_quantise(cs, 512, 1u << ns, m->Fs))) goto done;
    /* routes and fraction tables */
    uint32_t route_e[256];
    if ((st = bso_choose_routes(ceh, max_routes, m->route, &m->n_routes, route_e))) goto done;
    for (uint32_t r = 0; r < m->n_routes; r++)
        if ((st = bso_quantise(ceh + route_e[r] * 8, 8, 1u << nh, m->Fh[r]))) goto done;
    model_cums(m);
    out->n_routes = m->n_routes;
    /* pad word */
    uint32_t s_pad = 0;
    for (uint32_t s = 1; s < 512; s++)
        if (cs[s] > cs[s_pad]) s_pad = s;
    uint32_t h_pad = 0;
    if (m->route[s_pad & 0xFF] != 0xFF) {
        const uint32_t* row = m->Fh[m->route[s_pad & 0xFF]];
        for (uint32_t h = 1; h < 8; h++)
            if (row[h] > row[h_pad]) h_pad = h;
    }
    pad = (uint16_t)((s_pad << 7) | (h_pad << 4));

    /* serialize the model (4.3) */
    uint32_t n_present = 0;
    for (int s = 0; s < 512; s++) if (m->Fs[s]) n_present++;
    out->model_bytes = 260 + 4ull * n_present + 16ull * m->n_routes;
    out->model = (uint8_t*)calloc(1, out->model_bytes);
    if (!out->model) { st = BSO_E_NOMEM; goto done; }
    wr_u16(out->model, (uint16_t)n_present);
    uint64_t o = 4;
    for (int s = 0; s < 512; s++)
        if (m->Fs[s]) { wr_u16(out->model + o, (uint16_t)s); wr_u16(out->model + o + 2, (uint16_t)m->Fs[s]); o += 4; }
    memcpy(out->model + o, m->route, 256);
    o += 256;
    for (uint32_t r = 0; r < m->n_routes; r++)
        for (int h = 0; h < 8; h++) { wr_u16(out->model + o, (uint16_t)m->Fh[r][h]); o += 2; }

chunks:;
    /* nibble mode: constant when every weight has the same low nibble */
    out->nib_mode = 0x10u | (w[0] & 15u);
    for (uint64_t i = 1; i < n; i++)
        if ((w[i] & 15u) != (w[0] & 15u)) { out->nib_mode = 0; break; }
    const uint32_t nib_stored = out->nib_mode == 0;

    /* chunks */
    uint64_t C = 1ull << log2_chunk;
    out->n_chunks = (n + C - 1) / C;
    out->chunk = (uint8_t**)calloc(out->n_chunks, sizeof(uint8_t*));
    out->chunk_bytes = (uint64_t*)calloc(out->n_chunks, sizeof(uint64_t));
    out->chunk_words = (uint32_t*)calloc(out->n_chunks, sizeof(uint32_t));
    if (!out->chunk || !out->chunk_bytes || !out->chunk_words) { st = BSO_E_NOMEM; goto done; }
    out->coded_total = out->model_bytes + 16 * out->n_chunks;
    for (uint64_t c = 0; c < out->n_chunks; c++) {
        uint64_t base = c * C, nc = (n - base < C) ? n - base : C;
        uint32_t B = (uint32_t)((nc + 255) / 256), S = 8 * B;
        uint16_t* lw = (uint16_t*)malloc(sizeof(uint16_t) * S);
        uint8_t* em = (uint8_t*)malloc((size_t)LANES * S);
        uint16_t* wd = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)LANES * S);
        uint32_t* nib = (uint32_t*)calloc((size_t)LANES * B, sizeof(uint32_t));
        uint32_t states[LANES];
        if (!lw || !em || !wd || !nib) { free(lw); free(em); free(wd); free(nib); st = BSO_E_NOMEM; goto done; }
        for (uint32_t j = 0; j < LANES; j++) {
            for (uint32_t t = 0; t < S; t++) {
                uint64_t i = octet_index(t, j);
                lw[t] = (i < nc) ? w[base + i] : pad;
                nib[(size_t)(t >> 3) * LANES + j] |= (uint32_t)(lw[t] & 15u) << nibble_shift(t);
            }
            states[j] = lane_encode(m, lw, S, em + (size_t)j * S, wd + (size_t)j * S);
        }
        /* interleave: (t ascending, lane ascending) */
        uint32_t nw = 0;
        for (uint32_t t = 0; t < S; t++)
            for (uint32_t j = 0; j < LANES; j++) nw += em[(size_t)j * S + t];
        uint64_t bytes = align16(128 + 128ull * B * nib_stored + 2ull * nw);
        uint8_t* p = (uint8_t*)calloc(1, bytes);
        if (!p) { free(lw); free(em); free(wd); free(nib); st = BSO_E_NOMEM; goto done; }
        for (uint32_t j = 0; j < LANES; j++) wr_u32(p + 4 * j, states[j]);
        if (nib_stored)
            for (uint64_t k = 0; k < (uint64_t)LANES * B; k++) wr_u32(p + 128 + 4 * k, nib[k]);
        uint64_t q = 128 + 128ull * B * nib_stored;
        for (uint32_t t = 0; t < S; t++)
            for (uint32_t j = 0; j < LANES; j++)
                if (em[(size_t)j * S + t]) { wr_u16(p + q, wd[(size_t)j * S + t]); q += 2; }
        out->chunk[c] = p;
        out->chunk_bytes[c] = bytes;
        out->chunk_words[c] = nw;
        out->coded_total += bytes;
        free(lw); free(em); free(wd); free(nib);
    }
    st = BSO_OK;
done:
    if (m) model_free(m);
    free(m); free(cs); free(ceh); free(cj);
    if (st) blob_free(out);
    return st;
}

/* ------------------------------------------------------------------ */
/* Container writer: header, directory, names, then each tensor        */
/* ------------------------------------------------------------------ */
typedef struct {
    uint32_t kind;     /* 0: BF16 words (RANS or STORED chosen by the encoder); 2: RAW bytes */
    uint32_t ndim;
    uint64_t shape[8];
    uint64_t n_elems;  /* words for kind 0, bytes for kind 2 */
    const void* data;
    const char* name;
    uint32_t name_bytes;
    uint32_t reserved;
} bso_item;

typedef struct {
    uint32_t log2_chunk, ns, nh, max_routes, force_rans;
    uint32_t joint; /* 1: the JOINT kind instead of the factored RANS model */
    uint32_t nj;    /* JOINT precision, 8..13 */
} bso_params;

int bso_encode(const bso_item* items, uint32_t n_items, const bso_params* p, uint8_t** out, uint64_t* out_len) {
    if (!items && n_items) return BSO_E_ARG;
    if (!p || !out || !out_len) return BSO_E_ARG;
    if (p->log2_chunk < 8 || p->log2_chunk > 24 || p->ns < 1 || p->ns > 12 || p->nh < 3 || p->nh > 5 ||
        p->ns + p->nh > 16 || p->max_routes > 15 || p->joint > 1 || (p->joint && (p->nj < 8 || p->nj > 13)))
        return BSO_E_ARG;
    int st = BSO_OK;
    const uint32_t coded_kind = p->joint ? KIND_JOINT : KIND_RANS;
    rans_blob_t* blobs = (rans_blob_t*)calloc(n_items ? n_items : 1, sizeof(rans_blob_t));
    uint8_t* kinds = (uint8_t*)calloc(n_items ? n_items : 1, 1);
    if (!blobs || !kinds) { free(blobs); free(kinds); return BSO_E_NOMEM; }
    uint64_t names_bytes = 0;
    for (uint32_t k = 0; k < n_items; k++) {
        const bso_item* it = &items[k];
        uint64_t prod = 1;
        if (it->ndim > 8 || (it->kind != 0 && it->kind != 2) || (it->n_elems && !it->data)) { st = BSO_E_ARG; goto fail; }
        for (uint32_t d = 0; d < it->ndim; d++) prod *= it->shape[d];
        if (prod != it->n_elems) { st = BSO_E_ARG; goto fail; }
        names_bytes += it->name_bytes;
        if (it->kind == 2) { kinds[k] = KIND_RAW; continue; }
        if (it->n_elems > (1ull << 40)) { st = BSO_E_ARG; goto fail; }
        if (it->n_elems == 0) { kinds[k] = KIND_STORED; continue; }
        if (p->joint) { /* more distinct pairs than 2^nj slots: no JOINT table, so STORED */
            const uint16_t* w = (const uint16_t*)it->data;
            uint8_t* seen = (uint8_t*)calloc(JOINT_PAIRS, 1);
            uint32_t n_pairs = 0;
            if (!seen) { st = BSO_E_NOMEM; goto fail; }
            for (uint64_t i = 0; i < it->n_elems; i++)
                if (!seen[w[i] >> 4]) { seen[w[i] >> 4] = 1; n_pairs++; }
            free(seen);
            if (n_pairs > (1u << p->nj)) { kinds[k] = KIND_STORED; continue; }
        }
        if ((st = encode_rans((const uint16_t*)it->data, it->n_elems, p->log2_chunk, p->ns, p->nh, p->max_routes,
                              p->joint, p->nj, &blobs[k])))
            goto fail;
        if (!p->force_rans && blobs[k].coded_total >= 2 * it->n_elems) { kinds[k] = KIND_STORED; blob_free(&blobs[k]); }
        else kinds[k] = (uint8_t)coded_kind;
    }
    /* layout */
    uint64_t dir_off = HEADER_BYTES, names_off = align16(dir_off + (uint64_t)DIR_ENTRY_BYTES * n_items);
    uint64_t pos = align16(names_off + names_bytes);
    uint64_t* data_off = (uint64_t*)calloc(n_items ? n_items : 1, sizeof(uint64_t));
    uint64_t* model_off = (uint64_t*)calloc(n_items ? n_items : 1, sizeof(uint64_t));
    uint64_t** chunk_off = (uint64_t**)calloc(n_items ? n_items : 1, sizeof(uint64_t*));
    if (!data_off || !model_off || !chunk_off) { st = BSO_E_NOMEM; goto fail2; }
    for (uint32_t k = 0; k < n_items; k++) {
        if (is_coded(kinds[k])) {
            model_off[k] = pos;
            pos = align16(pos + blobs[k].model_bytes);
            data_off[k] = pos;
            pos = align16(pos + 16 * blobs[k].n_chunks);
            chunk_off[k] = (uint64_t*)calloc(blobs[k].n_chunks, sizeof(uint64_t));
            if (!chunk_off[k]) { st = BSO_E_NOMEM; goto fail2; }
            for (uint64_t c = 0; c < blobs[k].n_chunks; c++) { chunk_off[k][c] = pos; pos += blobs[k].chunk_bytes[c]; }
        } else {
            uint64_t bytes = (kinds[k] == KIND_STORED) ? 2 * items[k].n_elems : items[k].n_elems;
            data_off[k] = pos;
            pos = align16(pos + bytes);
        }
    }
    uint64_t total = pos;
    uint8_t* buf = (uint8_t*)calloc(1, total);
    if (!buf) { st = BSO_E_NOMEM; goto fail2; }
    memcpy(buf, "BF16RANS", 8);
    wr_u32(buf + 8, FORMAT_VERSION);
    wr_u32(buf + 12, HEADER_BYTES);
    wr_u32(buf + 16, n_items);
    wr_u32(buf + 20, DIR_ENTRY_BYTES);
    wr_u64(buf + 24, dir_off);
    wr_u64(buf + 32, names_off);
    wr_u64(buf + 40, names_bytes);
    wr_u64(buf + 48, total);
    uint64_t name_pos = 0;
    for (uint32_t k = 0; k < n_items; k++) {
        const bso_item* it = &items[k];
        uint8_t* d = buf + dir_off + (uint64_t)DIR_ENTRY_BYTES * k;
        d[0] = kinds[k];
        d[1] = (uint8_t)it->ndim;
        wr_u32(d + 8, (uint32_t)name_pos);
        wr_u32(d + 12, it->name_bytes);
        wr_u64(d + 16, it->n_elems);
        wr_u64(d + 64, bso_checksum(it->data, it->n_elems, it->kind == 2 ? 2 : 0));
        for (uint32_t dd = 0; dd < it->ndim; dd++) wr_u64(d + 80 + 8 * dd, it->shape[dd]);
        if (it->name_bytes) memcpy(buf + names_off + name_pos, it->name, it->name_bytes);
        name_pos += it->name_bytes;
        if (is_coded(kinds[k])) {
            const rans_blob_t* b = &blobs[k];
            d[2] = (uint8_t)p->log2_chunk;
            d[3] = LANES;
            d[4] = (uint8_t)(p->joint ? p->nj : p->ns);
            d[5] = (uint8_t)(p->joint ? 0 : p->nh);
            d[6] = (uint8_t)b->n_routes;
            d[7] = (uint8_t)b->nib_mode;
            wr_u64(d + 24, b->n_chunks);
            wr_u64(d + 32, model_off[k]);
            wr_u64(d + 40, b->model_bytes);
            wr_u64(d + 48, data_off[k]);
            wr_u64(d + 56, 16 * b->n_chunks);
            memcpy(buf + model_off[k], b->model, b->model_bytes);
            for (uint64_t c = 0; c < b->n_chunks; c++) {
                uint8_t* e = buf + data_off[k] + 16 * c;
                wr_u64(e, chunk_off[k][c]);
                wr_u32(e + 8, b->chunk_words[c]);
                memcpy(buf + chunk_off[k][c], b->chunk[c], b->chunk_bytes[c]);
            }
        } else {
            uint64_t bytes = (kinds[k] == KIND_STORED) ? 2 * it->n_elems : it->n_elems;
            wr_u64(d + 48, data_off[k]);
            wr_u64(d + 56, bytes);
            if (kinds[k] == KIND_STORED) {
                const uint16_t* w = (const uint16_t*)it->data;
                for (uint64_t i = 0; i < it->n_elems; i++) wr_u16(buf + data_off[k] + 2 * i, w[i]);
            } else if (bytes) {
                memcpy(buf + data_off[k], it->data, bytes);
            }
        }
    }
    *out = buf;
    *out_len = total;
fail2:
    if (chunk_off)
        for (uint32_t k = 0; k < n_items; k++) free(chunk_off[k]);
    free(chunk_off); free(model_off); free(data_off);
fail:
    for (uint32_t k = 0; k < n_items; k++) blob_free(&blobs[k]);
    free(blobs); free(kinds);
    return st;
}

void bso_free(void* p) { free(p); }

/* ------------------------------------------------------------------ */
/* Parser and validation of the byte layout                           */
/* ------------------------------------------------------------------ */
typedef struct {
    uint32_t kind, ndim, log2_chunk, lanes, ns, nh, n_routes, name_offset, name_bytes, nib_mode;
    uint64_t n_elems, n_chunks, model_offset, model_bytes, data_offset, data_bytes, checksum;
    uint64_t shape[8];
    uint64_t coded_bytes; /* RANS: model + chunk table + chunk payloads (padded); else data bytes */
} bso_tensor_info;

static int in_bounds(uint64_t off, uint64_t bytes, uint64_t len) { return off <= len && bytes <= len - off; }

static int parse_header(const uint8_t* b, uint64_t len, uint32_t* n_tensors) {
    if (!b || len < HEADER_BYTES) return BSO_E_FORMAT;
    if (memcmp(b, "BF16RANS", 8) != 0) return BSO_E_FORMAT;
    if (rd_u32(b + 8) != FORMAT_VERSION) return BSO_E_VERSION;
    if (rd_u32(b + 12) != HEADER_BYTES || rd_u32(b + 20) != DIR_ENTRY_BYTES || rd_u64(b + 56) != 0) return BSO_E_FORMAT;
    if (rd_u64(b + 48) != len) return BSO_E_SIZE;
    uint32_t nt = rd_u32(b + 16);
    uint64_t dir = rd_u64(b + 24), names = rd_u64(b + 32), names_bytes = rd_u64(b + 40);
    if (dir % 16 || names % 16) return BSO_E_FORMAT;
    if (!in_bounds(dir, (uint64_t)DIR_ENTRY_BYTES * nt, len) || !in_bounds(names, names_bytes, len)) return BSO_E_FORMAT;
    *n_tensors = nt;
    return BSO_OK;
}

/* Validates one directory entry, its model and its chunk table (not the streams). */
static int parse_entry(const uint8_t* b, uint64_t len, uint32_t idx, bso_tensor_info* ti) {
    uint32_t nt;
    int st = parse_header(b, len, &nt);
    if (st) return st;
    if (idx >= nt) return BSO_E_ARG;
    const uint8_t* d = b + rd_u64(b + 24) + (uint64_t)DIR_ENTRY_BYTES * idx;
    memset(ti, 0, sizeof(*ti));
    ti->kind = d[0]; ti->ndim = d[1]; ti->log2_chunk = d[2]; ti->lanes = d[3];
    ti->ns = d[4]; ti->nh = d[5]; ti->n_routes = d[6]; ti->nib_mode = d[7];
    ti->name_offset = rd_u32(d + 8); ti->name_bytes = rd_u32(d + 12);
    ti->n_elems = rd_u64(d + 16); ti->n_chunks = rd_u64(d + 24);
    ti->model_offset = rd_u64(d + 32); ti->model_bytes = rd_u64(d + 40);
    ti->data_offset = rd_u64(d + 48); ti->data_bytes = rd_u64(d + 56);
    ti->checksum = rd_u64(d + 64);
    for (int k = 0; k < 8; k++) ti->shape[k] = rd_u64(d + 80 + 8 * k);
    if (ti->ndim > 8 || ti->kind > 3) return BSO_E_FORMAT;
    if (rd_u64(d + 72) != 0) return BSO_E_FORMAT;
    if (!is_coded(ti->kind) && ti->nib_mode != 0) return BSO_E_FORMAT;
    for (uint32_t k = ti->ndim; k < 8; k++)
        if (ti->shape[k] != 0) return BSO_E_FORMAT;
    if ((uint64_t)ti->name_offset + ti->name_bytes > rd_u64(b + 40)) return BSO_E_FORMAT;
    unsigned __int128 prod = 1;
    for (uint32_t k = 0; k < ti->ndim; k++) { prod *= ti->shape[k]; if (prod > ((unsigned __int128)1 << 64)) return BSO_E_FORMAT; }
    if (prod != ti->n_elems) return BSO_E_FORMAT;
    if (ti->data_offset % 16 || !in_bounds(ti->data_offset, ti->data_bytes, len)) return BSO_E_FORMAT;
    if (ti->kind == KIND_STORED || ti->kind == KIND_RAW) {
        uint64_t want = (ti->kind == KIND_STORED) ? 2 * ti->n_elems : ti->n_elems;
        if (ti->kind == KIND_STORED && ti->n_elems > (1ull << 62)) return BSO_E_FORMAT;
        if (ti->data_bytes != want) return BSO_E_FORMAT;
        ti->coded_bytes = want;
        return BSO_OK;
    }
    /* RANS and JOINT */
    if (ti->lanes != LANES || ti->log2_chunk < 8 || ti->log2_chunk > 24) return BSO_E_FORMAT;
    if (ti->kind == KIND_JOINT) {
        if (ti->ns < 8 || ti->ns > 13 || ti->nh != 0 || ti->n_routes != 0) return BSO_E_FORMAT;
    } else if (ti->ns < 1 || ti->ns > 12 || ti->nh < 3 || ti->nh > 5 || ti->ns + ti->nh > 16 || ti->n_routes > 15) {
        return BSO_E_FORMAT;
    }
    if (ti->nib_mode != 0 && (ti->nib_mode & 0xF0u) != 0x10u) return BSO_E_FORMAT;
    if (ti->n_elems == 0 || ti->n_elems > (1ull << 40)) return BSO_E_FORMAT;
    uint64_t C = 1ull << ti->log2_chunk;
    if (ti->n_chunks != (ti->n_elems + C - 1) / C || ti->data_bytes != 16 * ti->n_chunks) return BSO_E_FORMAT;
    if (ti->model_offset % 16 || !in_bounds(ti->model_offset, ti->model_bytes, len)) return BSO_E_FORMAT;
    const uint8_t* mm = b + ti->model_offset;
    if (ti->kind == KIND_JOINT) { /* n_pairs, reserved, then (j, Fj) with j ascending, sum 2^nj */
        if (ti->model_bytes < 8) return BSO_E_FORMAT;
        uint32_t n_pairs = rd_u16(mm);
        if (n_pairs < 1 || n_pairs > JOINT_PAIRS || rd_u16(mm + 2) != 0) return BSO_E_FORMAT;
        if (ti->model_bytes != 4 + 4ull * n_pairs) return BSO_E_FORMAT;
        uint64_t sumj = 0;
        int prevj = -1;
        for (uint32_t k = 0; k < n_pairs; k++) {
            int j = rd_u16(mm + 4 + 4 * k);
            uint32_t q = rd_u16(mm + 6 + 4 * k);
            if (j <= prevj || j >= JOINT_PAIRS || q == 0) return BSO_E_FORMAT;
            prevj = j;
            sumj += q;
        }
        if (sumj != (1ull << ti->ns)) return BSO_E_FORMAT;
        goto chunk_table;
    }
    if (ti->model_bytes < 264) return BSO_E_FORMAT;
    uint32_t n_present = rd_u16(mm);
    if (n_present < 1 || n_present > 512 || rd_u16(mm + 2) != 0) return BSO_E_FORMAT;
    if (ti->model_bytes != 260 + 4ull * n_present + 16ull * ti->n_routes) return BSO_E_FORMAT;
    uint64_t sum = 0;
    int prev = -1;
    for (uint32_t k = 0; k < n_present; k++) {
        int s = rd_u16(mm + 4 + 4 * k);
        uint32_t q = rd_u16(mm + 6 + 4 * k);
        if (s <= prev || s > 511 || q == 0) return BSO_E_FORMAT;
        prev = s;
        sum += q;
    }
    if (sum != (1ull << ti->ns)) return BSO_E_FORMAT;
    const uint8_t* route = mm + 4 + 4 * n_present;
    for (int e = 0; e < 256; e++)
        if (route[e] != 0xFF && route[e] >= ti->n_routes) return BSO_E_FORMAT;
    for (uint32_t r = 0; r < ti->n_routes; r++) {
        sum = 0;
        for (int h = 0; h < 8; h++) sum += rd_u16(route + 256 + 16 * r + 2 * h);
        if (sum != (1ull << ti->nh)) return BSO_E_FORMAT;
    }
chunk_table:
    ti->coded_bytes = ti->model_bytes + ti->data_bytes;
    for (uint64_t c = 0; c < ti->n_chunks; c++) {
        const uint8_t* e = b + ti->data_offset + 16 * c;
        uint64_t off = rd_u64(e);
        uint32_t nw = rd_u32(e + 8);
        uint64_t nc = (ti->n_elems - c * C < C) ? ti->n_elems - c * C : C;
        uint64_t bytes = align16(128 + 128 * ((nc + 255) / 256) * (ti->nib_mode == 0) + 2ull * nw);
        if (off % 16 || rd_u32(e + 12) != 0 || !in_bounds(off, bytes, len)) return BSO_E_FORMAT;
        ti->coded_bytes += bytes;
    }
    return BSO_OK;
}

int bso_validate(const uint8_t* b, uint64_t len, uint32_t* n_tensors) {
    uint32_t nt;
    int st = parse_header(b, len, &nt);
    if (st) return st;
    for (uint32_t k = 0; k < nt; k++) {
        bso_tensor_info ti;
        if ((st = parse_entry(b, len, k, &ti))) return st;
    }
    if (n_tensors) *n_tensors = nt;
    return BSO_OK;
}

int bso_tensor_info_get(const uint8_t* b, uint64_t len, uint32_t idx, bso_tensor_info* ti) {
    if (!ti) return BSO_E_ARG;
    return parse_entry(b, len, idx, ti);
}

static int load_model(const uint8_t* b, const bso_tensor_info* ti, model_t* m) {
    memset(m, 0, sizeof(*m));
    const uint8_t* mm = b + ti->model_offset;
    if (ti->kind == KIND_JOINT) {
        m->joint = 1;
        m->nj = ti->ns;
        uint32_t n_pairs = rd_u16(mm);
        for (uint32_t k = 0; k < n_pairs; k++) m->Fj[rd_u16(mm + 4 + 4 * k)] = rd_u16(mm + 6 + 4 * k);
        return joint_build(m);
    }
    m->ns = ti->ns; m->nh = ti->nh; m->n_routes = ti->n_routes;
    uint32_t n_present = rd_u16(mm);
    m->n_present = n_present;
    for (uint32_t k = 0; k < n_present; k++) m->Fs[rd_u16(mm + 4 + 4 * k)] = rd_u16(mm + 6 + 4 * k);
    const uint8_t* route = mm + 4 + 4 * n_present;
    memcpy(m->route, route, 256);
    for (uint32_t r = 0; r < ti->n_routes; r++)
        for (int h = 0; h < 8; h++) m->Fh[r][h] = rd_u16(route + 256 + 16 * r + 2 * h);
    model_cums(m);
    return model_build_lookups(m);
}

/* ------------------------------------------------------------------ */
/* Decoder: lanes in ascending order take the words, step by step     */
/* ------------------------------------------------------------------ */
/* Decode chunk c of a RANS tensor into out (its weights only). Returns BSO_E_CORRUPT
 * when the stream is inconsistent. Every loop is bounded by the chunk's weight count. */
static int decode_chunk(const uint8_t* b, const bso_tensor_info* ti, const model_t* m, uint64_t c, uint16_t* out) {
    const uint8_t* e = b + ti->data_offset + 16 * c;
    const uint8_t* p = b + rd_u64(e);
    uint32_t nw = rd_u32(e + 8);
    uint64_t C = 1ull << ti->log2_chunk, base = c * C;
    uint64_t nc = (ti->n_elems - base < C) ? ti->n_elems - base : C;
    uint32_t B = (uint32_t)((nc + 255) / 256), S = 8 * B;
    uint32_t P = m->ns + m->nh, Mh = 1u << m->nh;
    const int nib_stored = ti->nib_mode == 0;
    const uint8_t* nib = p + 128;
    const uint8_t* words = p + 128 + 128ull * B * nib_stored;
    uint32_t x[LANES];
    int bad = 0;
    for (int j = 0; j < LANES; j++) {
        x[j] = rd_u32(p + 4 * j);
        if (x[j] < STATE_L) bad = 1;
    }
    if (bad) return BSO_E_CORRUPT;
    uint32_t pos = 0;
    for (uint32_t t = 0; t < S; t++) {
        for (uint32_t j = 0; j < LANES; j++) { /* lanes in ascending order take words */
            uint32_t s, h;
            if (m->joint) { /* the JOINT kind: x = Fj[j] * (x >> nj) + slot - cum(j) */
                uint32_t slot = x[j] & ((1u << m->nj) - 1u);
                uint32_t pj = m->j_of_slot[slot];
                s = pj >> 3;
                h = pj & 7u;
                x[j] = m->Fj[pj] * (x[j] >> m->nj) + (slot - m->cum_j[pj]);
            } else {
                uint32_t slot = x[j] & ((1u << P) - 1u);
                uint32_t js = slot >> m->nh, jh = slot & (Mh - 1u);
                s = m->s_of_slot[js];
                uint8_t r = m->route[s & 0xFF];
                uint32_t row = (r == 0xFF) ? m->n_routes : r, qh, ch;
                h = m->h_of_slot[(size_t)row * Mh + jh];
                frac_model(m, s & 0xFF, h, &qh, &ch);
                x[j] = m->Fs[s] * qh * (x[j] >> P) + (js - m->cum_s[s]) * qh + (jh - ch);
            }
            if (x[j] < STATE_L) {
                uint32_t wd = 0;
                if (pos < nw) wd = rd_u16(words + 2ull * pos); else bad = 1;
                pos++;
                x[j] = (x[j] << 16) | wd;
            }
            uint32_t u = nib_stored ? (rd_u32(nib + 4ull * ((t >> 3) * LANES + j)) >> nibble_shift(t)) & 15u
                                    : ti->nib_mode & 15u;
            uint64_t i = octet_index(t, j);
            if (i < nc) out[base + i] = (uint16_t)((s << 7) | (h << 4) | u);
        }
    }
    for (int j = 0; j < LANES; j++)
        if (x[j] != STATE_L) bad = 1;
    if (bad || pos != nw) return BSO_E_CORRUPT;
    return BSO_OK;
}

/* Decode chunks [c0, c1) of tensor idx (RANS), or the whole data (STORED/RAW, c0=c1=0
 * accepted), into out which holds the whole tensor (out_bytes = 2*n or n for RAW).
 * *bad_chunk = first corrupt chunk or -1. */
int bso_decode_chunks(const uint8_t* b, uint64_t len, uint32_t idx, uint64_t c0, uint64_t c1, void* out,
                      uint64_t out_bytes, int64_t* bad_chunk) {
    bso_tensor_info ti;
    int st = parse_entry(b, len, idx, &ti);
    if (bad_chunk) *bad_chunk = -1;
    if (st) return st;
    uint64_t want = (ti.kind == KIND_RAW) ? ti.n_elems : 2 * ti.n_elems;
    if (out_bytes != want || (want && !out)) return BSO_E_SIZE;
    if (!is_coded(ti.kind)) {
        if (ti.kind == KIND_STORED) {
            uint16_t* w = (uint16_t*)out;
            for (uint64_t i = 0; i < ti.n_elems; i++) w[i] = rd_u16(b + ti.data_offset + 2 * i);
        } else if (want) {
            memcpy(out, b + ti.data_offset, want);
        }
        return BSO_OK;
    }
    if (c0 > c1 || c1 > ti.n_chunks) return BSO_E_ARG;
    model_t* m = (model_t*)calloc(1, sizeof(model_t));
    if (!m) return BSO_E_NOMEM;
    if ((st = load_model(b, &ti, m))) { model_free(m); free(m); return st; }
    for (uint64_t c = c0; c < c1; c++) {
        int cs = decode_chunk(b, &ti, m, c, (uint16_t*)out);
        if (cs) { st = cs; if (bad_chunk && *bad_chunk < 0) *bad_chunk = (int64_t)c; }
    }
    model_free(m);
    free(m);
    return st;
}

/* Whole tensor, then the per-tensor checksum: a mismatch is BSO_E_CORRUPT
 * with *bad_chunk = -1 (no single chunk is to blame). */
int bso_decode(const uint8_t* b, uint64_t len, uint32_t idx, void* out, uint64_t out_bytes, int64_t* bad_chunk) {
    bso_tensor_info ti;
    int st = parse_entry(b, len, idx, &ti);
    if (st) return st;
    st = bso_decode_chunks(b, len, idx, 0, is_coded(ti.kind) ? ti.n_chunks : 0, out, out_bytes, bad_chunk);
    if (st) return st;
    if (bso_checksum(out, ti.n_elems, ti.kind == KIND_RAW ? 2 : 0) != ti.checksum) return BSO_E_CORRUPT;
    return BSO_OK;
}
