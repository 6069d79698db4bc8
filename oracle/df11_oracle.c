/*
 * DF11 oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded CPU encoder and decoder for the DFloat11
 * ("Dynamic-Length Float") container.  Only the test suite, the smoke check
 * and the benchmark's CPU-baseline / reference arm may load this library; the
 * product path (the CUDA library) never calls it and shares no code with it.
 *
 * Sources (page title, section):
 *   [DF11-summary] "DFloat11: compressao sem perda para inferencia em GPU que
 *                   reduz LLMs para 70% do tamanho" (news.hada.io summary)
 *   [DF11-abstract] "70% Size, 100% Accuracy: Lossless LLM Compression for
 *                   Efficient GPU Inference via Dynamic-Length Float"
 *
 * What each function follows:
 *   - field split / merge: [DF11-summary] "O espaco de compressao ainda
 *     disponivel no expoente" (1 sign bit, 8 exponent bits, 7 mantissa bits)
 *     and "O formato DFloat11" (sign+mantissa kept raw in PackedSignMantissa).
 *   - histogram, entropy: [DF11-summary] "O espaco de compressao ..." (Shannon
 *     entropy of the exponent field).
 *   - code lengths: [DF11-summary] "O formato DFloat11" (a Huffman tree over
 *     the exponent distribution) with the 32-bit length cap implied by
 *     "Kernel de GPU em 2 etapas e metadados auxiliares" (gaps fit in 5 bits
 *     because codes are at most 32 bits).  Read here as the optimal
 *     length-limited prefix code, computed with package-merge.
 *   - canonical codes, MSB-first bit packing, padding: readings of the format
 *     that the pages leave open (stated in the design notes as R3, R4, R6).
 *   - bit-serial decode: [DF11-summary] "Descompressao adaptada para
 *     inferencia em GPU" (the traditional bit-level walk of the Huffman tree).
 *   - Gaps, per-thread-block output positions, windowed decode:
 *     [DF11-summary] "Kernel de GPU em 2 etapas e metadados auxiliares".
 *
 * Parity pins: every function here is pinned by the CPU tests (exhaustive
 * split/merge, hand-worked golden stream, brute-force optimal lengths,
 * textbook Huffman cost, Kraft equality, entropy bound, windowed re-decode).
 * No function is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_CORRUPT 3
#define ORC_ERR_TOO_LARGE 4
#define ORC_ERR_CAPACITY 5

/* ------------------------------------------------------------------------ */
/* BF16 field split: bit 15 sign, bits 14..7 exponent, bits 6..0 mantissa.   */
/* PackedSignMantissa byte: bit 7 = sign, bits 6..0 = mantissa (reading R2). */
/* ------------------------------------------------------------------------ */
uint32_t oracle_exponent(uint32_t x) { return (x >> 7) & 0xFFu; }

uint32_t oracle_sign_mantissa(uint32_t x) {
    uint32_t sign = (x >> 15) & 1u;
    uint32_t mant = x & 0x7Fu;
    return (sign << 7) | mant;
}

uint32_t oracle_merge(uint32_t e, uint32_t sm) {
    uint32_t sign = (sm >> 7) & 1u;
    uint32_t mant = sm & 0x7Fu;
    return (sign << 15) | ((e & 0xFFu) << 7) | mant;
}

/* ------------------------------------------------------------------------ */
/* Histogram of the 8-bit exponent field and its Shannon entropy in bits.    */
/* ------------------------------------------------------------------------ */
void oracle_histogram(const uint16_t* x, uint64_t n, uint64_t* hist) {
    for (int s = 0; s < 256; s++) hist[s] = 0;
    for (uint64_t i = 0; i < n; i++) hist[oracle_exponent(x[i])] += 1;
}

double oracle_entropy_bits(const uint64_t* hist) {
    double total = 0.0;
    for (int s = 0; s < 256; s++) total += (double)hist[s];
    if (total <= 0.0) return 0.0;
    double h = 0.0;
    for (int s = 0; s < 256; s++) {
        if (hist[s] == 0) continue;
        double p = (double)hist[s] / total;
        h -= p * log2(p);
    }
    return h;
}

/* ------------------------------------------------------------------------ */
/* Optimal length-limited code lengths: package-merge (coin collector).      */
/*                                                                           */
/* Every present symbol owns one coin of each denomination 2^-d, d = 1..L,    */
/* worth its count.  The cheapest set of coins whose denominations add up to  */
/* (m - 1) gives the code lengths: a symbol's length is the number of its     */
/* coins taken.  Lists are built from the deepest denomination upwards: the   */
/* list at depth d is the merge of the depth-d leaf coins with the packages   */
/* formed by pairing consecutive items of the depth-(d+1) list.  At depth 1   */
/* the first 2(m-1) items are taken.                                          */
/*                                                                           */
/* Tie rule (reading R5, makes the result unique): leaves are ordered by      */
/* (count ascending, symbol ascending); when a leaf and a package weigh the   */
/* same, the leaf comes first.                                                */
/* ------------------------------------------------------------------------ */
typedef struct {
    uint64_t weight;
    int is_leaf;
    int symbol;   /* valid for leaves */
    int child_a;  /* index into the list one level deeper (packages) */
    int child_b;
} pm_item;

static void pm_expand(pm_item** lists, int depth, int idx, uint8_t* len_out) {
    pm_item* it = &lists[depth][idx];
    if (it->is_leaf) {
        len_out[it->symbol] += 1;
        return;
    }
    pm_expand(lists, depth + 1, it->child_a, len_out);
    pm_expand(lists, depth + 1, it->child_b, len_out);
}

int oracle_code_lengths(const uint64_t* hist, int max_len, uint8_t* len_out) {
    int syms[256];
    int m = 0;
    for (int s = 0; s < 256; s++) len_out[s] = 0;
    for (int s = 0; s < 256; s++)
        if (hist[s] > 0) syms[m++] = s;
    if (m == 0) return ORC_OK;
    if (max_len < 1 || max_len > 32) return ORC_ERR_ARG;
    if (m == 1) { /* one symbol: a single 1-bit code "0" (reading R12) */
        len_out[syms[0]] = 1;
        return ORC_OK;
    }
    if (max_len < 9 && (1 << max_len) < m) return ORC_ERR_ARG;

    /* insertion sort of the leaves by (count, symbol) */
    for (int i = 1; i < m; i++) {
        int v = syms[i];
        int j = i - 1;
        while (j >= 0 && (hist[syms[j]] > hist[v] ||
                          (hist[syms[j]] == hist[v] && syms[j] > v))) {
            syms[j + 1] = syms[j];
            j--;
        }
        syms[j + 1] = v;
    }

    pm_item* lists[34];
    int count[34];
    for (int d = 0; d < 34; d++) { lists[d] = NULL; count[d] = 0; }

    /* deepest list: the leaf coins alone */
    lists[max_len] = (pm_item*)calloc((unsigned)m, sizeof(pm_item));
    if (!lists[max_len]) return ORC_ERR_ARG;
    for (int i = 0; i < m; i++) {
        lists[max_len][i].weight = hist[syms[i]];
        lists[max_len][i].is_leaf = 1;
        lists[max_len][i].symbol = syms[i];
    }
    count[max_len] = m;

    for (int d = max_len - 1; d >= 1; d--) {
        int npk = count[d + 1] / 2;
        pm_item* out = (pm_item*)calloc((unsigned)(m + npk), sizeof(pm_item));
        if (!out) {
            for (int q = 0; q < 34; q++) free(lists[q]);
            return ORC_ERR_ARG;
        }
        int li = 0, pi = 0, k = 0;
        while (li < m || pi < npk) {
            uint64_t pw = 0;
            if (pi < npk)
                pw = lists[d + 1][2 * pi].weight + lists[d + 1][2 * pi + 1].weight;
            int take_leaf;
            if (li >= m) take_leaf = 0;
            else if (pi >= npk) take_leaf = 1;
            else take_leaf = (hist[syms[li]] <= pw); /* leaf first on ties */
            if (take_leaf) {
                out[k].weight = hist[syms[li]];
                out[k].is_leaf = 1;
                out[k].symbol = syms[li];
                li++;
            } else {
                out[k].weight = pw;
                out[k].is_leaf = 0;
                out[k].child_a = 2 * pi;
                out[k].child_b = 2 * pi + 1;
                pi++;
            }
            k++;
        }
        lists[d] = out;
        count[d] = k;
    }

    int take = 2 * (m - 1);
    int rc = ORC_OK;
    if (count[1] < take) rc = ORC_ERR_ARG;
    else
        for (int i = 0; i < take; i++) pm_expand(lists, 1, i, len_out);
    for (int d = 0; d < 34; d++) free(lists[d]);
    if (rc != ORC_OK)
        for (int s = 0; s < 256; s++) len_out[s] = 0;
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Canonical codes (reading R4): present symbols sorted by (length, value);   */
/* the first gets code 0, each next one (previous + 1) shifted left by the    */
/* length increase.                                                          */
/* ------------------------------------------------------------------------ */
int oracle_canonical_codes(const uint8_t* len, uint32_t* code_out) {
    int order[256];
    int m = 0;
    for (int s = 0; s < 256; s++) code_out[s] = 0;
    for (int l = 1; l <= 32; l++)
        for (int s = 0; s < 256; s++)
            if (len[s] == l) order[m++] = s;
    for (int s = 0; s < 256; s++)
        if (len[s] > 32) return ORC_ERR_ARG;
    if (m == 0) return ORC_OK;
    uint64_t code = 0;
    int prev_len = len[order[0]];
    for (int k = 0; k < m; k++) {
        int l = len[order[k]];
        if (k > 0) code = (code + 1) << (l - prev_len);
        if (code >> l) return ORC_ERR_ARG; /* lengths violate Kraft */
        code_out[order[k]] = (uint32_t)code;
        prev_len = l;
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Sizes of the container arrays (readings R6, R8-R11).                     */
/*   total_bits = sum of code lengths                                         */
/*   n_threads  = ceil(total_bits / 64)      (one 8-byte window per thread)   */
/*   n_blocks   = ceil(n_threads / T)                                         */
/*   bytes_exp  = 8*T*n_blocks + 16          (zero padding + guard)           */
/*   bytes_sm   = n rounded up to 16                                          */
/*   bytes_gaps = ceil(5*T*n_blocks/8) + 8, rounded up to 16                  */
/*   bytes_off  = 4*(n_blocks + 1)                                            */
/* ------------------------------------------------------------------------ */
typedef struct {
    uint64_t n_elems;
    uint64_t total_bits;
    uint64_t n_threads;
    uint64_t n_blocks;
    uint64_t bytes_exp;
    uint64_t bytes_sm;
    uint64_t bytes_gaps;
    uint64_t bytes_off;
} oracle_sizes;

static uint64_t round_up(uint64_t v, uint64_t m) { return (v + m - 1) / m * m; }

int oracle_sizes_for(const uint64_t* hist, const uint8_t* len, uint32_t T,
                     oracle_sizes* out) {
    if (T < 1) return ORC_ERR_ARG;
    uint64_t n = 0, bits = 0;
    for (int s = 0; s < 256; s++) {
        n += hist[s];
        if (hist[s] && len[s] == 0) return ORC_ERR_ARG;
        bits += hist[s] * (uint64_t)len[s];
    }
    if (n >= ((uint64_t)1 << 32)) return ORC_ERR_TOO_LARGE;
    out->n_elems = n;
    out->total_bits = bits;
    out->n_threads = (bits + 63) / 64;
    out->n_blocks = (out->n_threads + T - 1) / T;
    out->bytes_exp = 8 * (uint64_t)T * out->n_blocks + 16;
    out->bytes_sm = round_up(n, 16);
    out->bytes_gaps = round_up((5 * (uint64_t)T * out->n_blocks + 7) / 8 + 8, 16);
    out->bytes_off = 4 * (out->n_blocks + 1);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Bit helpers.  EncodedExponent is MSB-first (reading R3): stream bit p is   */
/* bit (7 - p%8) of byte p/8.  Gaps are 5-bit fields packed LSB-first         */
/* (reading R9): field t occupies stream bits 5t..5t+4, bit q of the array    */
/* being bit (q%8) of byte q/8.                                               */
/* ------------------------------------------------------------------------ */
static int get_bit_msb(const uint8_t* a, uint64_t p) { return (a[p >> 3] >> (7 - (p & 7))) & 1; }
static void set_bit_msb(uint8_t* a, uint64_t p) { a[p >> 3] |= (uint8_t)(0x80u >> (p & 7)); }

static uint32_t get_gap(const uint8_t* gaps, uint64_t t) {
    uint32_t g = 0;
    for (int k = 0; k < 5; k++) {
        uint64_t q = 5 * t + (uint64_t)k;
        g |= (uint32_t)((gaps[q >> 3] >> (q & 7)) & 1) << k;
    }
    return g;
}
static void put_gap(uint8_t* gaps, uint64_t t, uint32_t g) {
    for (int k = 0; k < 5; k++) {
        uint64_t q = 5 * t + (uint64_t)k;
        if ((g >> k) & 1) gaps[q >> 3] |= (uint8_t)(1u << (q & 7));
    }
}
uint32_t oracle_read_gap(const uint8_t* gaps, uint64_t t) { return get_gap(gaps, t); }

/* ------------------------------------------------------------------------ */
/* Encoder: EncodedExponent, PackedSignMantissa, Gaps, block offsets.        */
/*   gap[w]  = (first code start >= 64w, or total_bits if none) - 64w        */
/*   off[b]  = number of codes starting before bit 64*T*b, b = 0..n_blocks    */
/* ------------------------------------------------------------------------ */
int oracle_encode(const uint16_t* x, uint64_t n, const uint8_t* len, uint32_t T,
                  uint8_t* exp, uint64_t exp_cap, uint8_t* sm, uint64_t sm_cap,
                  uint8_t* gaps, uint64_t gaps_cap, uint32_t* off, uint64_t off_cap) {
    uint64_t hist[256];
    oracle_histogram(x, n, hist);
    oracle_sizes sz;
    int rc = oracle_sizes_for(hist, len, T, &sz);
    if (rc != ORC_OK) return rc;
    if (exp_cap < sz.bytes_exp || sm_cap < sz.bytes_sm || gaps_cap < sz.bytes_gaps ||
        off_cap < sz.n_blocks + 1)
        return ORC_ERR_CAPACITY;
    uint32_t code[256];
    rc = oracle_canonical_codes(len, code);
    if (rc != ORC_OK) return rc;

    memset(exp, 0, (size_t)sz.bytes_exp);
    memset(sm, 0, (size_t)sz.bytes_sm);
    memset(gaps, 0, (size_t)sz.bytes_gaps);
    memset(off, 0, (size_t)(sz.n_blocks + 1) * sizeof(uint32_t));

    /* codes, MSB first, and the raw sign+mantissa bytes */
    uint64_t p = 0;
    for (uint64_t i = 0; i < n; i++) {
        uint32_t e = oracle_exponent(x[i]);
        int l = len[e];
        for (int k = l - 1; k >= 0; k--) {
            if ((code[e] >> k) & 1u) set_bit_msb(exp, p);
            p++;
        }
        sm[i] = (uint8_t)oracle_sign_mantissa(x[i]);
    }
    if (p != sz.total_bits) return ORC_ERR_ARG;

    /* Gaps and block offsets from the code start positions */
    uint64_t w = 0, b = 0;
    p = 0;
    for (uint64_t i = 0; i < n; i++) {
        uint64_t start = p;
        while (w < sz.n_threads && 64 * w <= start) {
            uint64_t g = start - 64 * w;
            if (g > 31) return ORC_ERR_ARG;
            put_gap(gaps, w, (uint32_t)g);
            w++;
        }
        while (b <= sz.n_blocks && 64 * (uint64_t)T * b <= start) {
            off[b] = (uint32_t)i;
            b++;
        }
        p += len[oracle_exponent(x[i])];
    }
    while (w < sz.n_threads) {
        uint64_t g = sz.total_bits - 64 * w;
        if (g > 31) return ORC_ERR_ARG;
        put_gap(gaps, w, (uint32_t)g);
        w++;
    }
    while (b <= sz.n_blocks) {
        off[b] = (uint32_t)n;
        b++;
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Decoding trie built from the code table: the "traditional" decoder that   */
/* walks the Huffman tree one bit at a time.                                 */
/* ------------------------------------------------------------------------ */
#define TRIE_MAX_NODES (256 * 32 + 1) /* every prefix of every code, plus the root */
typedef struct {
    int child[TRIE_MAX_NODES][2]; /* node -> child node index, -1 = none */
    int symbol[TRIE_MAX_NODES];   /* leaf symbol, -1 for internal nodes   */
    int n_nodes;
} oracle_trie;

static int trie_build(const uint8_t* len, oracle_trie* tr) {
    uint32_t code[256];
    int rc = oracle_canonical_codes(len, code);
    if (rc != ORC_OK) return rc;
    tr->n_nodes = 1;
    tr->child[0][0] = tr->child[0][1] = -1;
    tr->symbol[0] = -1;
    for (int s = 0; s < 256; s++) {
        int l = len[s];
        if (l == 0) continue;
        int node = 0;
        for (int k = l - 1; k >= 0; k--) {
            int bit = (int)((code[s] >> k) & 1u);
            if (tr->symbol[node] >= 0) return ORC_ERR_ARG; /* not prefix-free */
            if (tr->child[node][bit] < 0) {
                if (tr->n_nodes >= TRIE_MAX_NODES) return ORC_ERR_ARG;
                int nn = tr->n_nodes++;
                tr->child[nn][0] = tr->child[nn][1] = -1;
                tr->symbol[nn] = -1;
                tr->child[node][bit] = nn;
            }
            node = tr->child[node][bit];
        }
        if (tr->symbol[node] >= 0 || tr->child[node][0] >= 0 || tr->child[node][1] >= 0)
            return ORC_ERR_ARG; /* not prefix-free */
        tr->symbol[node] = s;
    }
    return ORC_OK;
}

/* Decode one code starting at stream bit *p; codes may not run past limit. */
static int trie_decode_one(const oracle_trie* tr, const uint8_t* exp, uint64_t* p,
                           uint64_t limit, int* sym) {
    int node = 0;
    for (int depth = 0; depth < 32; depth++) {
        if (*p >= limit) return ORC_ERR_CORRUPT;
        int bit = get_bit_msb(exp, *p);
        *p += 1;
        node = tr->child[node][bit];
        if (node < 0) return ORC_ERR_CORRUPT;
        if (tr->symbol[node] >= 0) {
            *sym = tr->symbol[node];
            return ORC_OK;
        }
    }
    return ORC_ERR_CORRUPT;
}

/* Bit-serial decode of the whole stream; ignores Gaps and block offsets. */
int oracle_decode(const uint8_t* len, const uint8_t* exp, uint64_t total_bits,
                  const uint8_t* sm, uint64_t n, uint16_t* out) {
    oracle_trie* tr = (oracle_trie*)malloc(sizeof(oracle_trie));
    if (!tr) return ORC_ERR_ARG;
    int rc = trie_build(len, tr);
    uint64_t p = 0;
    for (uint64_t i = 0; i < n && rc == ORC_OK; i++) {
        int sym = 0;
        rc = trie_decode_one(tr, exp, &p, total_bits, &sym);
        if (rc == ORC_OK) out[i] = (uint16_t)oracle_merge((uint32_t)sym, sm[i]);
    }
    if (rc == ORC_OK && p != total_bits) rc = ORC_ERR_CORRUPT;
    free(tr);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Windowed decode: the work split of the two-phase GPU kernel, done         */
/* serially.  Thread w decodes every code that starts in its 64-bit window,   */
/* beginning at 64w + gap[w]; thread block b writes output from off[b] on.    */
/* Checks that (a) each window's decoding ends exactly where the next        */
/* window's first code starts, (b) every block produces off[b+1]-off[b]      */
/* symbols.  Decodes blocks [b0, b1); out receives elements off[b0]..off[b1]. */
/* ------------------------------------------------------------------------ */
int oracle_decode_windowed(const uint8_t* len, const uint8_t* exp, uint64_t total_bits,
                           const uint8_t* sm, const uint8_t* gaps, const uint32_t* off,
                           uint32_t T, uint64_t n_threads, uint64_t b0, uint64_t b1,
                           uint16_t* out) {
    oracle_trie* tr = (oracle_trie*)malloc(sizeof(oracle_trie));
    if (!tr) return ORC_ERR_ARG;
    int rc = trie_build(len, tr);
    uint64_t base = (b0 < b1) ? off[b0] : 0;
    for (uint64_t b = b0; b < b1 && rc == ORC_OK; b++) {
        uint64_t idx = off[b];
        for (uint64_t t = 0; t < T && rc == ORC_OK; t++) {
            uint64_t w = b * T + t;
            if (w >= n_threads) break;
            uint64_t p = 64 * w + get_gap(gaps, w);
            uint64_t end = 64 * (w + 1);
            if (end > total_bits) end = total_bits;
            while (p < end) {
                int sym = 0;
                rc = trie_decode_one(tr, exp, &p, total_bits, &sym);
                if (rc != ORC_OK) break;
                if (idx >= off[b + 1]) { rc = ORC_ERR_CORRUPT; break; }
                out[idx - base] = (uint16_t)oracle_merge((uint32_t)sym, sm[idx]);
                idx++;
            }
            if (rc != ORC_OK) break;
            /* the next window must start where this one stopped */
            if (w + 1 < n_threads && p != 64 * (w + 1) + get_gap(gaps, w + 1))
                rc = ORC_ERR_CORRUPT;
            if (w + 1 == n_threads && p != total_bits) rc = ORC_ERR_CORRUPT;
        }
        if (rc == ORC_OK && idx != off[b + 1]) rc = ORC_ERR_CORRUPT;
    }
    free(tr);
    return rc;
}
