/*
 * dfx_oracle.c -- plain, slow, single-threaded CPU oracle for the DFX1 codec.
 *
 * TEST INFRASTRUCTURE ONLY.  This file exists to check the CUDA codec.  Only the
 * test-suite, the package smoke check and the benchmark's CPU-baseline leg may
 * load it.  It shares no source, header, table or helper with the CUDA library
 * (lossless_entropy_coded_exponent_b200/csrc), and the CUDA library never calls it.
 *
 * What it computes.  The method is lossless entropy coding of BF16 weights:
 * weights of trained networks have a low-entropy value distribution, so a
 * variable-length code that gives frequent values short codes shrinks them
 * with bit-for-bit identical reconstruction
 *   ("DFloat11: lossless LLM compression for GPU", aikraft.ru blog, section 02
 *    "How DFloat11 works: entropy coding of the weights"; the ~1.5:1 figure of
 *    "From a Lossless (~1.5:1) Compression Algorithm for Llama2 7B Weights to
 *    Variable Precision, Variable Range, Compressed Numeric Data Types for CNNs
 *    and LLMs", abstract).
 * The pages leave the concrete code open.  This codec's reading, written out
 * step by step below, is:
 *   1. split every BF16 word into its 8-bit exponent and an 8-bit
 *      mantissa+sign byte: the 7 mantissa bits above one sign bit.  Elements
 *      2i and 2i+1 are partners and each byte carries its partner's sign (the
 *      last element of an odd-length tensor has none and keeps its own), so
 *      that a decoder rebuilds two weights with one 32-bit rotate;
 *   2. histogram the exponents;
 *   3. length-limited (max_len, default 24) Huffman code lengths by
 *      package-merge, ties broken by symbol value;
 *   4. canonical codes from the lengths;
 *   5. concatenate the codes MSB-first into 32-bit words;
 *   6. index: per chunk of K symbols its bit length, per group of G chunks its
 *      start bit: the small per-thread position records with which the GPU
 *      threads find where to read (DFloat11 blog, section 03, item 2).  The
 *      elements of a group (G*K of them) are cut into blocks of 8; block b
 *      belongs to chunk b mod G, so a chunk holds K/8 blocks spaced G blocks
 *      apart, and the codes are concatenated chunk after chunk;
 *   7. serialise the DFX1 container;
 *   8. decode bit by bit (canonical first-code/count walk), check the index
 *      against the walk, merge the two bytes back.
 * No step is blocked, fused or reordered beyond that list.
 * A second exponent coder (coder 1, tANS) replaces steps 3-5 and 8 with the
 * rules T1-T5 stated at the end of this file, and coder 2 adds rule T6 (two
 * interleaved tANS states per chunk) to them; everything else is shared.
 *
 * The container layout (all integers little-endian, every section starts at a
 * 16-byte boundary, every padding byte is zero):
 *   0   "DFX1"                                  magic
 *   4   u16 version = 1, u16 header_bytes = 64
 *   8   u64 n              number of BF16 elements
 *   16  u64 total_bits     length of the code stream in bits
 *   24  u64 total_bytes    size of the whole container
 *   32  u32 K              symbols per chunk (a multiple of 8)
 *   36  u32 G              chunks per group
 *   40  u32 n_chunk = G * n_group
 *   44  u32 n_group = ceil(n / (G * K))
 *   48  u64 off_m          byte offset of the sign+mantissa plane
 *   56  u32 max_len        code-length limit used by the encoder
 *   60  u32 reserved = 0
 *   64  u8  len[256]       code length of every exponent value (0 = unused)
 *   320 u64 gbase[n_group + 1]  start bit of each group, gbase[n_group] = total_bits
 *   .   u16 clen[n_chunk]       bit length of each chunk (0 for a chunk of the
 *                               last group that has no element)
 *   .   u8  m[n]                mantissa+sign bytes, element order:
 *                               m[x] = mantissa(x) * 2 + sign(partner(x)),
 *                               partner(x) = x ^ 1 if that is < n, else x
 *   .   u32 stream[...]         codes, bit k of the stream = bit (31 - k % 32)
 *                               of word k / 32; 4*ceil(total_bits/32) bytes
 *                               rounded up to 16, then 16 zero bytes of slack
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define DFXO_OK 0
#define DFXO_ERR_ARG 1
#define DFXO_ERR_CAPACITY 2
#define DFXO_ERR_CORRUPT 3

#define DFXO_HEADER_BYTES 64u
#define DFXO_LEN_OFFSET 64u
#define DFXO_GBASE_OFFSET 320u
#define DFXO_CODER_HUFFMAN 0u
#define DFXO_CODER_TANS 1u
#define DFXO_CODER_TANS2 2u /* tANS with two interleaved states per chunk (rule T6) */
#define DFXO_FREQ_OFFSET 64u
#define DFXO_TANS_GBASE_OFFSET 576u

/* ------------------------------------------------------------------ */
/* little-endian helpers (the container is little-endian by definition) */

static void put_u16(uint8_t *p, uint16_t v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }
static void put_u32(uint8_t *p, uint32_t v) { for (int i = 0; i < 4; i++) p[i] = (uint8_t)(v >> (8 * i)); }
static void put_u64(uint8_t *p, uint64_t v) { for (int i = 0; i < 8; i++) p[i] = (uint8_t)(v >> (8 * i)); }
static uint16_t get_u16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static uint32_t get_u32(const uint8_t *p) {
    uint32_t v = 0;
    for (int i = 3; i >= 0; i--) v = (v << 8) | p[i];
    return v;
}
static uint64_t get_u64(const uint8_t *p) {
    uint64_t v = 0;
    for (int i = 7; i >= 0; i--) v = (v << 8) | p[i];
    return v;
}
static uint64_t align16(uint64_t x) { return (x + 15u) & ~(uint64_t)15u; }

/* ------------------------------------------------------------------ */
/* Step 1: the split.  BF16 = sign(1) | exponent(8) | mantissa(7).  The other
 * byte of element x holds x's mantissa above its partner's sign:
 * mantissa(x) * 2 + sign(partner(x)).                                     */

uint8_t dfxo_exponent(uint16_t w) { return (uint8_t)((w >> 7) & 0xFF); }
uint64_t dfxo_partner(uint64_t x, uint64_t n) { return (x ^ 1u) < n ? (x ^ 1u) : x; }
uint8_t dfxo_sign_mantissa(uint16_t w, uint16_t partner) {
    return (uint8_t)(((w & 0x7F) << 1) | (partner >> 15));
}
/* e: x's exponent; m: x's byte; m_partner: the byte of x's partner */
uint16_t dfxo_merge(uint8_t e, uint8_t m, uint8_t m_partner) {
    return (uint16_t)(((uint16_t)(m_partner & 1) << 15) | ((uint16_t)e << 7) | (m >> 1));
}

/* ------------------------------------------------------------------ */
/* Step 2: histogram of the exponents ("frequent values get short codes",
 * DFloat11 blog, section 02).                                           */

int dfxo_histogram(const uint16_t *w, uint64_t n, uint64_t counts[256]) {
    for (int s = 0; s < 256; s++) counts[s] = 0;
    for (uint64_t i = 0; i < n; i++) counts[dfxo_exponent(w[i])]++;
    return DFXO_OK;
}

/* ------------------------------------------------------------------ */
/* Step 3: length-limited code lengths by package-merge.
 *
 * The coin-collector formulation: every used symbol is a coin of weight
 * count[s] at each of max_len denominations.  Start from the leaves sorted by
 * (count, symbol); max_len - 1 times, pair consecutive items of the current
 * list into packages (a trailing odd item is dropped) and merge the packages
 * with the leaves by weight, a leaf ahead of a package of equal weight.  The
 * first 2m - 2 items of the last list are selected; the length of a symbol is
 * the number of times its leaf occurs inside the selected items, packages
 * expanded down to their leaves.
 * One used symbol (m = 1): that symbol and a phantom partner (symbol 1 if the
 * used one is 0, else symbol 0) both get length 1; the phantom never occurs. */

typedef struct {
    uint64_t w;   /* weight */
    int sym;      /* leaf: symbol value; package: -1 */
    int a, b;     /* package: indices of its two children in the previous list */
} pm_item;

static int leaf_before(const pm_item *x, const pm_item *y) {
    /* leaf order: count ascending, then symbol ascending */
    if (x->w != y->w) return x->w < y->w;
    return x->sym < y->sym;
}

static void pm_expand(pm_item **lists, int level, int idx, uint8_t len[256]) {
    const pm_item *it = &lists[level][idx];
    if (it->sym >= 0) {
        len[it->sym]++;
        return;
    }
    pm_expand(lists, level - 1, it->a, len);
    pm_expand(lists, level - 1, it->b, len);
}

int dfxo_code_lengths(const uint64_t counts[256], uint32_t max_len, uint8_t len[256]) {
    pm_item leaves[256];
    int m = 0;
    for (int s = 0; s < 256; s++) len[s] = 0;
    for (int s = 0; s < 256; s++)
        if (counts[s] > 0) {
            leaves[m].w = counts[s];
            leaves[m].sym = s;
            leaves[m].a = leaves[m].b = -1;
            m++;
        }
    if (m == 0) return DFXO_OK;
    if (m == 1) {
        int s0 = leaves[0].sym;
        len[s0] = 1;
        len[s0 == 0 ? 1 : 0] = 1;
        return DFXO_OK;
    }
    if (max_len < 1 || max_len > 32) return DFXO_ERR_ARG;
    if (max_len < 9 && (1u << max_len) < (uint32_t)m) return DFXO_ERR_ARG; /* no prefix code exists */

    /* insertion sort of the leaves by (count, symbol) */
    for (int i = 1; i < m; i++) {
        pm_item x = leaves[i];
        int j = i - 1;
        while (j >= 0 && leaf_before(&x, &leaves[j])) {
            leaves[j + 1] = leaves[j];
            j--;
        }
        leaves[j + 1] = x;
    }

    int L = (int)max_len;
    pm_item **lists = (pm_item **)calloc((size_t)L, sizeof(pm_item *));
    int *sizes = (int *)calloc((size_t)L, sizeof(int));
    if (!lists || !sizes) { free(lists); free(sizes); return DFXO_ERR_ARG; }
    lists[0] = (pm_item *)malloc(sizeof(pm_item) * (size_t)m);
    memcpy(lists[0], leaves, sizeof(pm_item) * (size_t)m);
    sizes[0] = m;
    for (int j = 1; j < L; j++) {
        int np = sizes[j - 1] / 2;
        pm_item *pk = (pm_item *)malloc(sizeof(pm_item) * (size_t)(np > 0 ? np : 1));
        for (int k = 0; k < np; k++) {
            pk[k].w = lists[j - 1][2 * k].w + lists[j - 1][2 * k + 1].w;
            pk[k].sym = -1;
            pk[k].a = 2 * k;
            pk[k].b = 2 * k + 1;
        }
        lists[j] = (pm_item *)malloc(sizeof(pm_item) * (size_t)(m + np));
        int i = 0, k = 0, o = 0;
        while (i < m || k < np) {
            if (k >= np || (i < m && leaves[i].w <= pk[k].w))
                lists[j][o++] = leaves[i++];
            else
                lists[j][o++] = pk[k++];
        }
        sizes[j] = o;
        free(pk);
    }
    int take = 2 * m - 2;
    int rc = DFXO_OK;
    if (sizes[L - 1] < take) rc = DFXO_ERR_ARG;
    else
        for (int t = 0; t < take; t++) pm_expand(lists, L - 1, t, len);
    for (int j = 0; j < L; j++) free(lists[j]);
    free(lists);
    free(sizes);
    return rc;
}

/* ------------------------------------------------------------------ */
/* Step 4: canonical codes.  Walk the used symbols in (length, symbol)
 * order; the first gets code 0, each next one the previous code plus one,
 * shifted left by the growth in length.                                 */

int dfxo_canonical_codes(const uint8_t len[256], uint32_t code[256]) {
    uint32_t c = 0;
    int prev = -1;
    for (int s = 0; s < 256; s++) code[s] = 0;
    for (int l = 1; l <= 32; l++)
        for (int s = 0; s < 256; s++) {
            if (len[s] != l) continue;
            if (prev < 0) c = 0;
            else c = (c + 1) << (l - prev);
            code[s] = c;
            prev = l;
        }
    return DFXO_OK;
}

/* ------------------------------------------------------------------ */
/* Layout rules.                                                        */

static int params_ok(uint64_t n, uint32_t K, uint32_t G, uint32_t max_len) {
    if (n >= ((uint64_t)1 << 32)) return 0;
    if (max_len < 1 || max_len > 24) return 0;
    if (K < 8 || K % 8 != 0 || G < 1) return 0;
    if ((uint64_t)K * max_len > 65535u) return 0; /* a chunk length must fit in u16 */
    return 1;
}

/* (0 for parameters no container can have, so that sizing never divides by zero) */
static uint64_t n_groups(uint64_t n, uint32_t K, uint32_t G) {
    return (G == 0 || K == 0) ? 0 : (n + (uint64_t)G * K - 1) / ((uint64_t)G * K);
}

/* Element of position `pos` (0..K-1) in chunk `lane` of group g: the group's
 * elements form blocks of 8, block b belongs to chunk b mod G. */
static uint64_t chunk_element(uint64_t g, uint32_t lane, uint32_t pos, uint32_t K, uint32_t G) {
    return g * G * K + ((uint64_t)(pos / 8) * G + lane) * 8 + pos % 8;
}
/* The sections after the code section are the same for both coders; only the
 * code section's size (len[256] for coder 0, freq[256] for coder 1) moves them. */
static int is_tans(uint32_t coder) { return coder == DFXO_CODER_TANS || coder == DFXO_CODER_TANS2; }
static uint64_t gbase_of(uint32_t coder) { return is_tans(coder) ? DFXO_TANS_GBASE_OFFSET : DFXO_GBASE_OFFSET; }
static uint64_t off_clen_of(uint64_t ng, uint32_t coder) { return align16(gbase_of(coder) + 8 * (ng + 1)); }
static uint64_t off_m_of(uint64_t nc, uint64_t ng, uint32_t coder) { return align16(off_clen_of(ng, coder) + 2 * nc); }
static uint64_t off_stream_of(uint64_t n, uint64_t nc, uint64_t ng, uint32_t coder) {
    return align16(off_m_of(nc, ng, coder) + n);
}
static uint64_t stream_bytes_of(uint64_t total_bits) { return align16(4 * ((total_bits + 31) / 32)) + 16; }

static uint64_t container_bytes_of(uint64_t n, uint32_t K, uint32_t G, uint64_t total_bits, uint32_t coder) {
    uint64_t ng = n_groups(n, K, G), nc = ng * G;
    return off_stream_of(n, nc, ng, coder) + stream_bytes_of(total_bits);
}
uint64_t dfxo_container_bytes(uint64_t n, uint32_t K, uint32_t G, uint64_t total_bits) {
    return container_bytes_of(n, K, G, total_bits, DFXO_CODER_HUFFMAN);
}

/* ------------------------------------------------------------------ */
/* Steps 5-7: stream, index, container.                                 */

static void put_bits(uint8_t *stream, uint64_t pos, uint32_t code, uint32_t l) {
    /* bit k of the stream is bit (31 - k % 32) of little-endian word k / 32 */
    for (uint32_t b = 0; b < l; b++) {
        uint32_t bit = (code >> (l - 1 - b)) & 1u;
        uint64_t k = pos + b;
        uint64_t word = k / 32;
        uint32_t within = 31u - (uint32_t)(k % 32);
        uint8_t *byte = stream + 4 * word + within / 8; /* little-endian word: byte i holds bits 8i..8i+7 */
        if (bit) *byte |= (uint8_t)(1u << (within % 8));
    }
}

static uint32_t get_bit(const uint8_t *stream, uint64_t k) {
    uint64_t word = k / 32;
    uint32_t within = 31u - (uint32_t)(k % 32);
    return (stream[4 * word + within / 8] >> (within % 8)) & 1u;
}

int dfxo_encode(const uint16_t *w, uint64_t n, uint32_t K, uint32_t G, uint32_t max_len,
                uint8_t *out, uint64_t cap, uint64_t *out_bytes) {
    if (!params_ok(n, K, G, max_len) || max_len < 8) return DFXO_ERR_ARG;
    uint64_t counts[256];
    uint8_t len[256];
    uint32_t code[256];
    dfxo_histogram(w, n, counts);
    int rc = dfxo_code_lengths(counts, max_len, len);
    if (rc) return rc;
    dfxo_canonical_codes(len, code);

    uint64_t total_bits = 0;
    for (uint64_t i = 0; i < n; i++) total_bits += len[dfxo_exponent(w[i])];
    uint64_t ng = n_groups(n, K, G), nc = ng * G;
    uint64_t total = dfxo_container_bytes(n, K, G, total_bits);
    if (out_bytes) *out_bytes = total;
    if (cap < total) return DFXO_ERR_CAPACITY;
    memset(out, 0, (size_t)total);

    memcpy(out, "DFX1", 4);
    put_u16(out + 4, 1);
    put_u16(out + 6, DFXO_HEADER_BYTES);
    put_u64(out + 8, n);
    put_u64(out + 16, total_bits);
    put_u64(out + 24, total);
    put_u32(out + 32, K);
    put_u32(out + 36, G);
    put_u32(out + 40, (uint32_t)nc);
    put_u32(out + 44, (uint32_t)ng);
    put_u64(out + 48, off_m_of(nc, ng, 0));
    put_u32(out + 56, max_len);
    put_u32(out + 60, 0);
    memcpy(out + DFXO_LEN_OFFSET, len, 256);

    /* stream in chunk order, index: chunk bit lengths and group start bits */
    uint8_t *gbase = out + DFXO_GBASE_OFFSET;
    uint8_t *clen = out + off_clen_of(ng, 0);
    uint8_t *mplane = out + off_m_of(nc, ng, 0);
    uint8_t *stream = out + off_stream_of(n, nc, ng, 0);
    uint64_t pos = 0;
    for (uint64_t g = 0; g < ng; g++) {
        put_u64(gbase + 8 * g, pos);
        for (uint32_t lane = 0; lane < G; lane++) {
            uint64_t start = pos;
            for (uint32_t k = 0; k < K; k++) {
                uint64_t x = chunk_element(g, lane, k, K, G);
                if (x >= n) break;
                uint8_t e = dfxo_exponent(w[x]);
                put_bits(stream, pos, code[e], len[e]);
                pos += len[e];
            }
            put_u16(clen + 2 * (g * G + lane), (uint16_t)(pos - start));
        }
    }
    put_u64(gbase + 8 * ng, pos);
    for (uint64_t i = 0; i < n; i++) mplane[i] = dfxo_sign_mantissa(w[i], w[dfxo_partner(i, n)]);
    return DFXO_OK;
}

uint64_t dfxo_max_container_bytes(uint64_t n, uint32_t K, uint32_t G) {
    /* An optimal length-limited code never costs more than the 8-bit
     * fixed-length code (feasible because max_len >= 8); the one-symbol
     * phantom code costs 1 bit per element. */
    return dfxo_container_bytes(n, K, G, 8 * n);
}

/* ------------------------------------------------------------------ */
/* Step 8: decode.  Validate everything, then walk the stream one bit at a
 * time: a code of length l is complete when its value minus the first
 * canonical code of length l is below the number of codes of length l.    */

static int decode_tans(const uint8_t *c, uint64_t bytes, uint16_t *w, uint64_t n_cap, uint64_t *n_out);

int dfxo_decode(const uint8_t *c, uint64_t bytes, uint16_t *w, uint64_t n_cap, uint64_t *n_out) {
    if (bytes >= DFXO_HEADER_BYTES && memcmp(c, "DFX1", 4) == 0 && is_tans(get_u32(c + 60)))
        return decode_tans(c, bytes, w, n_cap, n_out);
    if (bytes < DFXO_GBASE_OFFSET + 8) return DFXO_ERR_CORRUPT;
    if (memcmp(c, "DFX1", 4) != 0) return DFXO_ERR_CORRUPT;
    if (get_u16(c + 4) != 1 || get_u16(c + 6) != DFXO_HEADER_BYTES) return DFXO_ERR_CORRUPT;
    uint64_t n = get_u64(c + 8);
    uint64_t total_bits = get_u64(c + 16);
    uint64_t total = get_u64(c + 24);
    uint32_t K = get_u32(c + 32), G = get_u32(c + 36);
    uint32_t max_len = get_u32(c + 56);
    if (!params_ok(n, K, G, max_len)) return DFXO_ERR_CORRUPT;
    if (get_u32(c + 60) != 0) return DFXO_ERR_CORRUPT;
    uint64_t ng = n_groups(n, K, G), nc = ng * G;
    if (get_u32(c + 40) != nc || get_u32(c + 44) != ng) return DFXO_ERR_CORRUPT;
    if (get_u64(c + 48) != off_m_of(nc, ng, 0)) return DFXO_ERR_CORRUPT;
    if (total_bits > (uint64_t)max_len * n) return DFXO_ERR_CORRUPT;
    if (total != dfxo_container_bytes(n, K, G, total_bits) || total > bytes) return DFXO_ERR_CORRUPT;
    if (n_out) *n_out = n;
    if (n > n_cap) return DFXO_ERR_CAPACITY;

    /* code lengths: at most max_len; Kraft sum exactly 1 when n > 0, no code when n = 0 */
    const uint8_t *len = c + DFXO_LEN_OFFSET;
    uint64_t kraft = 0;
    for (int s = 0; s < 256; s++) {
        if (len[s] > max_len) return DFXO_ERR_CORRUPT;
        if (len[s]) kraft += (uint64_t)1 << (24 - len[s]);
    }
    if (n > 0 && kraft != ((uint64_t)1 << 24)) return DFXO_ERR_CORRUPT;
    if (n == 0 && kraft != 0) return DFXO_ERR_CORRUPT;

    /* canonical decoding tables: count and first code per length, symbols in (length, symbol) order */
    uint32_t count[33] = {0}, first[33] = {0}, index_of_first[33] = {0};
    uint8_t sorted[256];
    int ns = 0;
    for (int l = 1; l <= 24; l++)
        for (int s = 0; s < 256; s++)
            if (len[s] == l) {
                if (count[l] == 0) index_of_first[l] = (uint32_t)ns;
                count[l]++;
                sorted[ns++] = (uint8_t)s;
            }
    {
        uint32_t code = 0;
        int prev = -1;
        for (int l = 1; l <= 24; l++) {
            if (count[l] == 0) continue;
            if (prev < 0) code = 0;
            else code = (code + 1) << (l - prev);   /* code held the last code of length prev */
            first[l] = code;
            code += count[l] - 1;
            prev = l;
        }
    }

    const uint8_t *gbase = c + DFXO_GBASE_OFFSET;
    const uint8_t *clen = c + off_clen_of(ng, 0);
    const uint8_t *mplane = c + off_m_of(nc, ng, 0);
    const uint8_t *stream = c + off_stream_of(n, nc, ng, 0);

    /* every padding byte must be zero */
    for (uint64_t b = DFXO_GBASE_OFFSET + 8 * (ng + 1); b < off_clen_of(ng, 0); b++) if (c[b]) return DFXO_ERR_CORRUPT;
    for (uint64_t b = off_clen_of(ng, 0) + 2 * nc; b < off_m_of(nc, ng, 0); b++) if (c[b]) return DFXO_ERR_CORRUPT;
    for (uint64_t b = off_m_of(nc, ng, 0) + n; b < off_stream_of(n, nc, ng, 0); b++) if (c[b]) return DFXO_ERR_CORRUPT;
    if (get_u64(gbase) != 0 || get_u64(gbase + 8 * ng) != total_bits) return DFXO_ERR_CORRUPT;

    uint64_t pos = 0;
    for (uint64_t g = 0; g < ng; g++) {
        if (get_u64(gbase + 8 * g) != pos) return DFXO_ERR_CORRUPT;
        for (uint32_t lane = 0; lane < G; lane++) {
            uint64_t chunk_start = pos;
            for (uint32_t k = 0; k < K; k++) {
                uint64_t x = chunk_element(g, lane, k, K, G);
                if (x >= n) break;
                uint32_t code = 0;
                int l = 0, found = -1;
                while (l < 24) {
                    if (pos >= total_bits) return DFXO_ERR_CORRUPT;
                    code = (code << 1) | get_bit(stream, pos);
                    pos++;
                    l++;
                    if (count[l] && code >= first[l] && code - first[l] < count[l]) {
                        found = sorted[index_of_first[l] + (code - first[l])];
                        break;
                    }
                }
                if (found < 0) return DFXO_ERR_CORRUPT;
                w[x] = dfxo_merge((uint8_t)found, mplane[x], mplane[dfxo_partner(x, n)]);
            }
            if (get_u16(clen + 2 * (g * G + lane)) != pos - chunk_start) return DFXO_ERR_CORRUPT;
        }
    }
    if (pos != total_bits) return DFXO_ERR_CORRUPT;
    /* stream bits after total_bits, the rounding words and the slack are zero */
    for (uint64_t k = total_bits; k < 32 * ((total_bits + 31) / 32); k++) if (get_bit(stream, k)) return DFXO_ERR_CORRUPT;
    for (uint64_t b = 4 * ((total_bits + 31) / 32); b < stream_bytes_of(total_bits); b++) if (stream[b]) return DFXO_ERR_CORRUPT;
    return DFXO_OK;
}

/* ================================================================== */
/* Coder 1: tabled asymmetric numeral systems (tANS) for the exponents.
 *
 * One page names ANS as the entropy coder of its compressed number formats'
 * hardware decoder ("From a Lossless (~1.5:1) Compression Algorithm for Llama2
 * 7B Weights to Variable Precision, Variable Range, Compressed Numeric Data
 * Types for CNNs and LLMs", abstract) without giving a construction.  This
 * coder is the published tabled variant (J. Duda, "Asymmetric numeral
 * systems", 2013) with these rules, each a reading of this codec:
 *   T1. frequencies: M = 2^R (R = table_log, 4..12).  Every used exponent s
 *       gets f[s] = counts[s] * M / n rounded half up, at least 1; then the
 *       largest f (the smallest symbol among equal ones) takes the whole
 *       shortfall to M, or gives up an excess one unit at a time, until the
 *       f sum to M.  More used exponents than M: no table (argument error);
 *   T2. spread: list every symbol f[s] times in symbol order; occurrence i
 *       goes to table slot (i * step) mod M, step = M/2 + M/8 + 3 (odd, so
 *       for M >= 16, so every slot is hit once; the stride of Y. Collet's FSE
 *       coder);
 *   T3. states: the slots of symbol s, in ascending slot order, are numbered
 *       k = f[s], f[s] + 1, ..., 2 f[s] - 1;
 *   T4. a chunk's symbols are encoded from its last to its first, starting
 *       from state X = M: for symbol s take the nb >= 0 with
 *       f[s] <= X >> nb < 2 f[s], emit the low nb bits of X, and move to
 *       X = M + the slot of s numbered X >> nb.  The chunk's bits are the
 *       final X - M (R bits), then the emitted fields in symbol order
 *       (first symbol's first), each MSB-first; an empty chunk has no bits;
 *   T5. decoding a chunk: x = its first R bits; for each symbol, slot x holds
 *       symbol s with number k; with nb = R - floor(log2 k), x becomes
 *       k * 2^nb + (the next nb bits) - M.  After the last symbol x is 0.
 *   T6. (coder 2) two interleaved states: a chunk's symbols at even positions
 *       (0, 2, ...) are coded by state A, those at odd positions by state B,
 *       each by T4 on its own, both starting from X = M, the chunk still
 *       taken from its last symbol to its first; the chunk's bits are A's
 *       final X - M (R bits), B's final X - M (R bits), then every symbol's
 *       field in symbol order.  Decoding (T5 per state) reads A's and B's start
 *       states, then decodes symbol i with the state of i's parity; both
 *       states end at 0.  A lane's two table lookups per symbol pair are then
 *       independent, which halves the decoder's chain of dependent loads; the
 *       price is R more bits per chunk.
 * The container is the DFX1 layout with u32 coder = 1 (2 for T6) at offset 60,
 * the table log in the max_len word (offset 56), u16 freq[256] at offset 64
 * and the group start bits at offset 576; the chunks, groups and blocks are
 * those of coder 0.                                                      */

static int tans_params_ok(uint64_t n, uint32_t K, uint32_t G, uint32_t R, uint32_t ways) {
    if (n >= ((uint64_t)1 << 32)) return 0;
    if (R < 4 || R > 12) return 0;
    if (K < 8 || K % 8 != 0 || G < 1) return 0;
    if ((uint64_t)(K + ways) * R > 65535u) return 0; /* a chunk length must fit in u16 */
    return 1;
}

/* T1 */
int dfxo_tans_normalize(const uint64_t counts[256], uint32_t R, uint32_t f[256]) {
    if (R < 4 || R > 12) return DFXO_ERR_ARG;
    const uint64_t M = (uint64_t)1 << R;
    uint64_t n = 0, used = 0;
    for (int s = 0; s < 256; s++) {
        f[s] = 0;
        if (counts[s] >= ((uint64_t)1 << 40)) return DFXO_ERR_ARG;
        n += counts[s];
        used += counts[s] > 0;
    }
    if (n == 0) return DFXO_OK;
    if (used > M) return DFXO_ERR_ARG;
    uint64_t sum = 0;
    for (int s = 0; s < 256; s++) {
        if (!counts[s]) continue;
        uint64_t q = (2 * counts[s] * M + n) / (2 * n);
        f[s] = (uint32_t)(q ? q : 1);
        sum += f[s];
    }
    while (sum != M) {
        int big = 0;
        for (int s = 1; s < 256; s++)
            if (f[s] > f[big]) big = s;
        if (sum < M) {
            f[big] += (uint32_t)(M - sum);
            sum = M;
        } else { /* sum > M >= used, so f[big] >= 2 */
            f[big] -= 1;
            sum -= 1;
        }
    }
    return DFXO_OK;
}

/* T2 and T3: slot_sym[j] and slot_k[j] for the M slots.  f must sum to M. */
int dfxo_tans_tables(const uint32_t f[256], uint32_t R, uint8_t *slot_sym, uint32_t *slot_k) {
    if (R < 4 || R > 12) return DFXO_ERR_ARG;
    const uint32_t M = 1u << R;
    uint64_t sum = 0;
    for (int s = 0; s < 256; s++) sum += f[s];
    if (sum != M) return DFXO_ERR_ARG;
    const uint32_t step = (M >> 1) + (M >> 3) + 3;
    uint32_t i = 0;
    for (int s = 0; s < 256; s++)
        for (uint32_t r = 0; r < f[s]; r++, i++) slot_sym[(i * step) & (M - 1)] = (uint8_t)s;
    uint32_t next[256];
    for (int s = 0; s < 256; s++) next[s] = f[s];
    for (uint32_t j = 0; j < M; j++) slot_k[j] = next[slot_sym[j]]++;
    return DFXO_OK;
}

/* T4 (ways = 1) or T6 (ways = 2) for one chunk of cnt symbols e[]: its bit
 * length; when stream is not NULL the bits are also written from stream bit
 * `pos` on.  enc[cs[s] + k - f[s]] is the slot of s numbered k; v and nb hold
 * cnt fields.  Symbol i is coded by state i mod ways. */
static uint64_t tans_chunk(const uint32_t f[256], const uint32_t cs[256], const uint32_t *enc, uint32_t R,
                           uint32_t ways, const uint8_t *e, uint32_t cnt, uint8_t *stream, uint64_t pos, uint32_t *v,
                           uint8_t *nb) {
    if (cnt == 0) return 0;
    const uint32_t M = 1u << R;
    uint32_t X[2] = {M, M};
    uint64_t bits = (uint64_t)R * ways;
    for (uint32_t i = cnt; i-- > 0;) {
        const uint32_t s = e[i], st = i % ways;
        uint32_t b = 0;
        while ((X[st] >> b) >= 2 * f[s]) b++;
        v[i] = X[st] & ((1u << b) - 1u);
        nb[i] = (uint8_t)b;
        bits += b;
        X[st] = M + enc[cs[s] + (X[st] >> b) - f[s]];
    }
    if (stream) {
        for (uint32_t st = 0; st < ways; st++) {
            put_bits(stream, pos, X[st] - M, R);
            pos += R;
        }
        for (uint32_t i = 0; i < cnt; i++) {
            put_bits(stream, pos, v[i], nb[i]);
            pos += nb[i];
        }
    }
    return bits;
}

/* T4 (ways = 1) or T6 (ways = 2) for one chunk of cnt symbols with a given
 * frequency table f (summing to M): writes the chunk's bits MSB-first from bit 0
 * of `out` (zeroed by the caller, at least R * (cnt + ways) bits long) and
 * returns their number. */
int dfxo_tans_encode_chunk_ways(const uint32_t f[256], uint32_t R, uint32_t ways, const uint8_t *syms, uint32_t cnt,
                                uint8_t *out, uint64_t *bits) {
    if (R < 4 || R > 12 || ways < 1 || ways > 2) return DFXO_ERR_ARG;
    const uint32_t M = 1u << R;
    uint32_t cs[256], run = 0;
    for (int s = 0; s < 256; s++) {
        cs[s] = run;
        run += f[s];
    }
    for (uint32_t i = 0; i < cnt; i++)
        if (f[syms[i]] == 0) return DFXO_ERR_ARG;
    uint8_t *slot_sym = (uint8_t *)malloc(M);
    uint32_t *slot_k = (uint32_t *)malloc(4 * (size_t)M), *enc = (uint32_t *)malloc(4 * (size_t)M);
    uint32_t *v = (uint32_t *)malloc(4 * (size_t)(cnt + 1));
    uint8_t *nb = (uint8_t *)malloc(cnt + 1);
    int rc = DFXO_ERR_ARG;
    if (slot_sym && slot_k && enc && v && nb && dfxo_tans_tables(f, R, slot_sym, slot_k) == DFXO_OK) {
        for (uint32_t j = 0; j < M; j++) enc[cs[slot_sym[j]] + slot_k[j] - f[slot_sym[j]]] = j;
        *bits = tans_chunk(f, cs, enc, R, ways, syms, cnt, out, 0, v, nb);
        rc = DFXO_OK;
    }
    free(slot_sym);
    free(slot_k);
    free(enc);
    free(v);
    free(nb);
    return rc;
}

int dfxo_tans_encode_chunk(const uint32_t f[256], uint32_t R, const uint8_t *syms, uint32_t cnt, uint8_t *out,
                           uint64_t *bits) {
    return dfxo_tans_encode_chunk_ways(f, R, 1, syms, cnt, out, bits);
}

uint64_t dfxo_tans_container_bytes(uint64_t n, uint32_t K, uint32_t G, uint64_t total_bits) {
    return container_bytes_of(n, K, G, total_bits, DFXO_CODER_TANS);
}

uint64_t dfxo_tans_max_container_bytes(uint64_t n, uint32_t K, uint32_t G, uint32_t R) {
    /* a field is at most R bits (k >= 1), plus R bits of state per chunk */
    uint64_t nc = n_groups(n, K, G) * G;
    return container_bytes_of(n, K, G, (uint64_t)R * (n + nc), DFXO_CODER_TANS);
}

uint64_t dfxo_tans2_max_container_bytes(uint64_t n, uint32_t K, uint32_t G, uint32_t R) {
    /* T6: two states per chunk */
    uint64_t nc = n_groups(n, K, G) * G;
    return container_bytes_of(n, K, G, (uint64_t)R * (n + 2 * nc), DFXO_CODER_TANS2);
}

/* The symbols of chunk `lane` of group g, in chunk order; returns how many. */
static uint32_t chunk_symbols(const uint16_t *w, uint64_t n, uint64_t g, uint32_t lane, uint32_t K, uint32_t G,
                              uint8_t *e) {
    uint32_t cnt = 0;
    for (uint32_t k = 0; k < K; k++) {
        uint64_t x = chunk_element(g, lane, k, K, G);
        if (x >= n) break;
        e[cnt++] = dfxo_exponent(w[x]);
    }
    return cnt;
}

static int encode_tans_ways(const uint16_t *w, uint64_t n, uint32_t K, uint32_t G, uint32_t R, uint32_t ways,
                            uint8_t *out, uint64_t cap, uint64_t *out_bytes) {
    if (!tans_params_ok(n, K, G, R, ways)) return DFXO_ERR_ARG;
    const uint32_t coder = ways == 2 ? DFXO_CODER_TANS2 : DFXO_CODER_TANS;
    const uint32_t M = 1u << R;
    uint64_t counts[256];
    uint32_t f[256], cs[256];
    dfxo_histogram(w, n, counts);
    int rc = dfxo_tans_normalize(counts, R, f);
    if (rc) return rc;
    uint8_t *slot_sym = (uint8_t *)malloc(M);
    uint32_t *slot_k = (uint32_t *)malloc(4 * (size_t)M), *enc = (uint32_t *)malloc(4 * (size_t)M);
    uint32_t *v = (uint32_t *)malloc(4 * (size_t)K);
    uint8_t *e = (uint8_t *)malloc(K), *nb = (uint8_t *)malloc(K);
    if (!slot_sym || !slot_k || !enc || !v || !e || !nb) {
        rc = DFXO_ERR_ARG;
        goto done;
    }
    {
        uint32_t run = 0;
        for (int s = 0; s < 256; s++) {
            cs[s] = run;
            run += f[s];
        }
    }
    if (n > 0) {
        dfxo_tans_tables(f, R, slot_sym, slot_k);
        for (uint32_t j = 0; j < M; j++) enc[cs[slot_sym[j]] + slot_k[j] - f[slot_sym[j]]] = j;
    }
    uint64_t ng = n_groups(n, K, G), nc = ng * G;
    uint64_t total_bits = 0;
    for (uint64_t g = 0; g < ng; g++)
        for (uint32_t lane = 0; lane < G; lane++) {
            uint32_t cnt = chunk_symbols(w, n, g, lane, K, G, e);
            total_bits += tans_chunk(f, cs, enc, R, ways, e, cnt, NULL, 0, v, nb);
        }
    uint64_t total = container_bytes_of(n, K, G, total_bits, coder);
    if (out_bytes) *out_bytes = total;
    if (cap < total) {
        rc = DFXO_ERR_CAPACITY;
        goto done;
    }
    memset(out, 0, (size_t)total);
    memcpy(out, "DFX1", 4);
    put_u16(out + 4, 1);
    put_u16(out + 6, DFXO_HEADER_BYTES);
    put_u64(out + 8, n);
    put_u64(out + 16, total_bits);
    put_u64(out + 24, total);
    put_u32(out + 32, K);
    put_u32(out + 36, G);
    put_u32(out + 40, (uint32_t)nc);
    put_u32(out + 44, (uint32_t)ng);
    put_u64(out + 48, off_m_of(nc, ng, coder));
    put_u32(out + 56, R);
    put_u32(out + 60, coder);
    for (int s = 0; s < 256; s++) put_u16(out + DFXO_FREQ_OFFSET + 2 * s, (uint16_t)f[s]);
    {
        uint8_t *gbase = out + DFXO_TANS_GBASE_OFFSET;
        uint8_t *clen = out + off_clen_of(ng, coder);
        uint8_t *mplane = out + off_m_of(nc, ng, coder);
        uint8_t *stream = out + off_stream_of(n, nc, ng, coder);
        uint64_t pos = 0;
        for (uint64_t g = 0; g < ng; g++) {
            put_u64(gbase + 8 * g, pos);
            for (uint32_t lane = 0; lane < G; lane++) {
                uint32_t cnt = chunk_symbols(w, n, g, lane, K, G, e);
                uint64_t bits = tans_chunk(f, cs, enc, R, ways, e, cnt, stream, pos, v, nb);
                put_u16(clen + 2 * (g * G + lane), (uint16_t)bits);
                pos += bits;
            }
        }
        put_u64(gbase + 8 * ng, pos);
        for (uint64_t i = 0; i < n; i++) mplane[i] = dfxo_sign_mantissa(w[i], w[dfxo_partner(i, n)]);
    }
    rc = DFXO_OK;
done:
    free(slot_sym);
    free(slot_k);
    free(enc);
    free(v);
    free(e);
    free(nb);
    return rc;
}

int dfxo_encode_tans(const uint16_t *w, uint64_t n, uint32_t K, uint32_t G, uint32_t R, uint8_t *out, uint64_t cap,
                     uint64_t *out_bytes) {
    return encode_tans_ways(w, n, K, G, R, 1, out, cap, out_bytes);
}

int dfxo_encode_tans2(const uint16_t *w, uint64_t n, uint32_t K, uint32_t G, uint32_t R, uint8_t *out, uint64_t cap,
                      uint64_t *out_bytes) {
    return encode_tans_ways(w, n, K, G, R, 2, out, cap, out_bytes);
}

/* T5 (T6 for coder 2), with every header field, the frequency table, the index
 * and the padding checked. */
static int decode_tans(const uint8_t *c, uint64_t bytes, uint16_t *w, uint64_t n_cap, uint64_t *n_out) {
    if (bytes < DFXO_TANS_GBASE_OFFSET + 8) return DFXO_ERR_CORRUPT;
    if (get_u16(c + 4) != 1 || get_u16(c + 6) != DFXO_HEADER_BYTES) return DFXO_ERR_CORRUPT;
    const uint32_t coder = get_u32(c + 60), ways = coder == DFXO_CODER_TANS2 ? 2u : 1u;
    uint64_t n = get_u64(c + 8), total_bits = get_u64(c + 16), total = get_u64(c + 24);
    uint32_t K = get_u32(c + 32), G = get_u32(c + 36), R = get_u32(c + 56);
    if (!tans_params_ok(n, K, G, R, ways)) return DFXO_ERR_CORRUPT;
    uint64_t ng = n_groups(n, K, G), nc = ng * G;
    if (get_u32(c + 40) != nc || get_u32(c + 44) != ng) return DFXO_ERR_CORRUPT;
    if (get_u64(c + 48) != off_m_of(nc, ng, coder)) return DFXO_ERR_CORRUPT;
    if (total_bits > (uint64_t)R * (n + ways * nc)) return DFXO_ERR_CORRUPT;
    if (total != container_bytes_of(n, K, G, total_bits, coder) || total > bytes) return DFXO_ERR_CORRUPT;
    if (n_out) *n_out = n;
    if (n > n_cap) return DFXO_ERR_CAPACITY;

    const uint32_t M = 1u << R;
    uint32_t f[256];
    uint64_t sum = 0;
    for (int s = 0; s < 256; s++) {
        f[s] = get_u16(c + DFXO_FREQ_OFFSET + 2 * s);
        sum += f[s];
    }
    if (sum != (n > 0 ? M : 0)) return DFXO_ERR_CORRUPT;
    uint8_t *slot_sym = (uint8_t *)malloc(M);
    uint32_t *slot_k = (uint32_t *)malloc(4 * (size_t)M);
    int rc = DFXO_ERR_CORRUPT;
    if (!slot_sym || !slot_k) goto done;
    if (n > 0) dfxo_tans_tables(f, R, slot_sym, slot_k);

    const uint8_t *gbase = c + DFXO_TANS_GBASE_OFFSET;
    const uint8_t *clen = c + off_clen_of(ng, coder);
    const uint8_t *mplane = c + off_m_of(nc, ng, coder);
    const uint8_t *stream = c + off_stream_of(n, nc, ng, coder);
    for (uint64_t b = DFXO_TANS_GBASE_OFFSET + 8 * (ng + 1); b < off_clen_of(ng, coder); b++)
        if (c[b]) goto done;
    for (uint64_t b = off_clen_of(ng, coder) + 2 * nc; b < off_m_of(nc, ng, coder); b++)
        if (c[b]) goto done;
    for (uint64_t b = off_m_of(nc, ng, coder) + n; b < off_stream_of(n, nc, ng, coder); b++)
        if (c[b]) goto done;
    if (get_u64(gbase) != 0 || get_u64(gbase + 8 * ng) != total_bits) goto done;

    uint64_t pos = 0;
    for (uint64_t g = 0; g < ng; g++) {
        if (get_u64(gbase + 8 * g) != pos) goto done;
        for (uint32_t lane = 0; lane < G; lane++) {
            uint64_t chunk_start = pos;
            uint32_t x[2] = {0, 0};
            for (uint32_t k = 0; k < K; k++) {
                uint64_t xe = chunk_element(g, lane, k, K, G);
                if (xe >= n) break;
                if (k == 0) /* the chunk's first R bits (per state): the decoder's start states */
                    for (uint32_t st = 0; st < ways; st++)
                        for (uint32_t b = 0; b < R; b++) {
                            if (pos >= total_bits) goto done;
                            x[st] = (x[st] << 1) | get_bit(stream, pos++);
                        }
                uint32_t *xs = &x[k % ways]; /* T6: symbol k's state */
                uint32_t s = slot_sym[*xs], kk = slot_k[*xs], nbits = R, t = kk;
                while (t >>= 1) nbits--;
                uint32_t val = 0;
                for (uint32_t b = 0; b < nbits; b++) {
                    if (pos >= total_bits) goto done;
                    val = (val << 1) | get_bit(stream, pos++);
                }
                *xs = (kk << nbits) + val - M;
                w[xe] = dfxo_merge((uint8_t)s, mplane[xe], mplane[dfxo_partner(xe, n)]);
            }
            if (x[0] != 0 || x[1] != 0) goto done; /* every state ends in the encoder's start state */
            if (get_u16(clen + 2 * (g * G + lane)) != pos - chunk_start) goto done;
        }
    }
    if (pos != total_bits) goto done;
    for (uint64_t k = total_bits; k < 32 * ((total_bits + 31) / 32); k++)
        if (get_bit(stream, k)) goto done;
    for (uint64_t b = 4 * ((total_bits + 31) / 32); b < stream_bytes_of(total_bits); b++)
        if (stream[b]) goto done;
    rc = DFXO_OK;
done:
    free(slot_sym);
    free(slot_k);
    return rc;
}
