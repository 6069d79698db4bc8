// Host side of the DF11 library: error reporting, the length-limited code
// builder, canonical codes, header validation and the decode-table builder.
// Sources: "DFloat11: compressao sem perda para inferencia em GPU que reduz
// LLMs para 70% do tamanho" -- "O formato DFloat11" (Huffman code over the
// exponents), "Decodificacao com LUT hierarquica" (compact decode tables),
// "Kernel de GPU em 2 etapas e metadados auxiliares" (8-byte windows, 5-bit
// gaps, 32-bit codes at most, per-thread-block output positions).
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "df11_internal.h"

namespace df11 {

static thread_local char g_err[512] = "";

df11_status fail(df11_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return st;
}

bool canonical_codes(const uint8_t* len, uint32_t* code) {
    // count per length, then the first code of each length, then hand out
    // codes in increasing value order inside each length
    uint64_t bl_count[34] = {0};
    for (int s = 0; s < 256; s++) {
        code[s] = 0;
        if (len[s] > 32) return false;
        if (len[s]) bl_count[len[s]]++;
    }
    uint64_t next[34] = {0};
    uint64_t c = 0;
    for (int l = 1; l <= 32; l++) {
        c = (c + bl_count[l - 1]) << 1;
        next[l] = c;
    }
    for (int s = 0; s < 256; s++) {
        int l = len[s];
        if (!l) continue;
        uint64_t v = next[l]++;
        if (v >> l) return false;  // more codes than the length allows
        code[s] = uint32_t(v);
    }
    return true;
}

void fill_sizes(df11_header* h) {
    const uint64_t T = h->threads_per_block;
    h->n_threads = (h->total_bits + 63) / 64;
    h->n_blocks = (h->n_threads + T - 1) / T;
    h->bytes_exp = 8 * T * h->n_blocks + 16;
    h->bytes_sm = (h->n_elems + 15) & ~uint64_t(15);
    h->bytes_gaps = align16((5 * T * h->n_blocks + 7) / 8 + 8);
    h->bytes_off = 4 * (h->n_blocks + 1);
    h->bytes_lut = kLutBytes;
}

// Kraft sum in units of 2^-32; returns false on lengths > 32.
static bool kraft_units(const uint8_t* len, uint64_t* units, int* n_present) {
    uint64_t u = 0;
    int m = 0;
    for (int s = 0; s < 256; s++) {
        if (!len[s]) continue;
        if (len[s] > 32) return false;
        u += uint64_t(1) << (32 - len[s]);
        m++;
    }
    *units = u;
    *n_present = m;
    return true;
}

}  // namespace df11

using namespace df11;

// Decoded exponents are staged rotated right by one bit (bit 0 moves to bit
// 7): the two bytes of a BF16 value are then bit-selects of the rotated
// exponent and the sign+mantissa byte (high: sign | e >> 1, low:
// (e & 1) << 7 | mantissa).
static uint8_t rotate_symbol(uint8_t e) { return uint8_t((e >> 1) | (e << 7)); }

extern "C" {

int df11_version(void) { return DF11_VERSION; }

const char* df11_last_error(void) { return g_err; }

// Package-merge for optimal length-limited prefix codes.  Each present symbol
// has one coin per depth 1..L (value = its count); the cheapest coins whose
// depths' weights 2^-d sum to m-1 give the lengths.  The list of depth d is
// the depth-d coins merged with pairs of consecutive depth-(d+1) items.
// Instead of expanding the chosen packages, count down: if the first k items
// of depth d hold j leaves, those are the j lightest symbols (the merge keeps
// leaf order), each gains one bit, and the k - j packages stand for the first
// 2(k - j) items of depth d+1.
df11_status df11_code_lengths(const uint64_t* hist, uint32_t max_code_len, uint8_t* code_len) {
    if (!hist || !code_len) return fail(DF11_ERR_INVALID, "df11_code_lengths: null pointer");
    std::memset(code_len, 0, 256);
    int sym[256];
    int m = 0;
    for (int s = 0; s < 256; s++)
        if (hist[s]) sym[m++] = s;
    if (m == 0) return DF11_OK;
    if (max_code_len < 1 || max_code_len > 32)
        return fail(DF11_ERR_INVALID, "df11_code_lengths: max_code_len %u outside 1..32", max_code_len);
    if (m == 1) {
        code_len[sym[0]] = 1;
        return DF11_OK;
    }
    const int L = int(max_code_len);
    if (L < 9 && (1 << L) < m)
        return fail(DF11_ERR_INVALID, "df11_code_lengths: %d values do not fit in %d-bit codes", m, L);
    // lighter first; equal counts: lower value first
    std::sort(sym, sym + m, [&](int a, int b) { return hist[a] != hist[b] ? hist[a] < hist[b] : a < b; });

    // is_leaf[d][i]: item i of the depth-d list is a leaf coin.  A list holds
    // the m leaves and at most m - 1 packages (25 KB on the stack: no
    // allocation)
    uint8_t is_leaf[33][512];
    uint64_t wbuf[2][512];
    uint64_t* prev = wbuf[0];
    uint64_t* cur = wbuf[1];
    size_t n_prev = size_t(m), n_d1 = 0;
    for (int i = 0; i < m; i++) {
        prev[i] = hist[sym[i]];
        is_leaf[L][i] = 1;
    }
    if (L == 1) n_d1 = size_t(m);
    for (int d = L - 1; d >= 1; d--) {
        const size_t npk = n_prev / 2;
        size_t li = 0, pi = 0, nc = 0;
        while (li < size_t(m) || pi < npk) {
            const bool have_pk = pi < npk;
            const uint64_t pw = have_pk ? prev[2 * pi] + prev[2 * pi + 1] : 0;
            if (li < size_t(m) && (!have_pk || hist[sym[li]] <= pw)) {
                cur[nc] = hist[sym[li++]];
                is_leaf[d][nc++] = 1;
            } else {
                cur[nc] = pw;
                is_leaf[d][nc++] = 0;
                pi++;
            }
        }
        std::swap(prev, cur);
        n_prev = nc;
        if (d == 1) n_d1 = nc;
    }
    size_t k = size_t(2 * (m - 1));
    if (n_d1 < k) return fail(DF11_ERR_INVALID, "df11_code_lengths: too few items");
    for (int d = 1; d <= L && k; d++) {
        size_t j = 0;
        for (size_t i = 0; i < k; i++) j += is_leaf[d][i];
        for (size_t i = 0; i < j; i++) code_len[sym[i]]++;
        k = 2 * (k - j);
    }
    return DF11_OK;
}

df11_status df11_header_init(df11_header* hdr, const uint8_t* code_len, uint64_t n_elems,
                             uint64_t total_bits, uint32_t threads_per_block,
                             uint32_t max_code_len, const uint64_t* seg_counts,
                             uint32_t n_segs) {
    if (!hdr || !code_len) return fail(DF11_ERR_INVALID, "df11_header_init: null pointer");
    const uint32_t T = threads_per_block;
    if (T < 32 || T > 1024 || (T & (T - 1)))
        return fail(DF11_ERR_INVALID, "threads_per_block %u is not a power of two in 32..1024", T);
    if (max_code_len < 1 || max_code_len > 32)
        return fail(DF11_ERR_INVALID, "max_code_len %u outside 1..32", max_code_len);
    if (n_elems >= (uint64_t(1) << 32))
        return fail(DF11_ERR_TOO_LARGE, "n_elems %llu does not fit the 32-bit block offsets",
                    (unsigned long long)n_elems);
    if (n_segs < 1 || n_segs > DF11_MAX_SEGMENTS)
        return fail(DF11_ERR_INVALID, "n_segments %u outside 1..%d", n_segs, DF11_MAX_SEGMENTS);
    uint64_t units;
    int m;
    if (!kraft_units(code_len, &units, &m))
        return fail(DF11_ERR_INVALID, "code length above 32");
    for (int s = 0; s < 256; s++)
        if (code_len[s] > max_code_len)
            return fail(DF11_ERR_INVALID, "code length %u above max_code_len %u", code_len[s], max_code_len);
    if (n_elems > 0 && m == 0) return fail(DF11_ERR_INVALID, "empty code table for a non-empty stream");
    if (m == 1 && units != (uint64_t(1) << 31))
        return fail(DF11_ERR_INVALID, "a single present value must have the 1-bit code");
    if (m >= 2 && units != (uint64_t(1) << 32))
        return fail(DF11_ERR_INVALID, "code lengths are not a complete prefix code (Kraft sum != 1)");
    if (n_elems && (total_bits < n_elems || total_bits > 32 * n_elems))
        return fail(DF11_ERR_INVALID, "total_bits %llu inconsistent with %llu elements",
                    (unsigned long long)total_bits, (unsigned long long)n_elems);
    if (!n_elems && total_bits) return fail(DF11_ERR_INVALID, "bits without elements");

    std::memset(hdr, 0, sizeof(*hdr));
    hdr->version = DF11_VERSION;
    hdr->window_bytes = DF11_WINDOW_BYTES;
    hdr->threads_per_block = T;
    hdr->max_code_len = max_code_len;
    hdr->n_elems = n_elems;
    hdr->total_bits = total_bits;
    std::memcpy(hdr->code_len, code_len, 256);
    hdr->n_segments = n_segs;
    uint64_t acc = 0;
    for (uint32_t k = 0; k < n_segs; k++) {
        hdr->seg_elem_off[k] = acc;
        acc += seg_counts ? seg_counts[k] : n_elems;
    }
    hdr->seg_elem_off[n_segs] = acc;
    if (acc != n_elems) return fail(DF11_ERR_INVALID, "segment counts do not add up to n_elems");
    fill_sizes(hdr);
    return DF11_OK;
}

// Decode tables for hdr->code_len, in the layout of df11_internal.h.
df11_status df11_build_lut(const df11_header* hdr, void* h_lut, uint64_t cap) {
    if (!hdr || !h_lut) return fail(DF11_ERR_INVALID, "df11_build_lut: null pointer");
    if (cap < kLutBytes) return fail(DF11_ERR_CAPACITY, "df11_build_lut: need %llu bytes",
                                     (unsigned long long)kLutBytes);
    const uint8_t* len = hdr->code_len;
    uint32_t code[256];
    if (!canonical_codes(len, code)) return fail(DF11_ERR_INVALID, "code lengths overflow");

    uint8_t* blob = static_cast<uint8_t*>(h_lut);
    std::memset(blob, 0, kLutBytes);
    LutHeader lh{};
    lh.magic = kLutMagic;
    lh.peek_bits = kPeekBits;
    lh.escape = kEscape;

    // per-length counts and first codes
    uint64_t count[34] = {0}, first[34] = {0};
    for (int s = 0; s < 256; s++)
        if (len[s]) count[len[s]]++;
    uint64_t c = 0;
    for (int l = 1; l <= 32; l++) {
        c = (c + count[l - 1]) << 1;
        first[l] = c;
    }
    // symbols sorted by (length, value); base = codes shorter than l
    uint8_t* syms = blob + kLutOffSyms;
    uint32_t base[34] = {0};
    int n = 0;
    lh.min_len = 0;
    lh.max_len = 0;
    for (int l = 1; l <= 32; l++) {
        base[l] = uint32_t(n);
        for (int s = 0; s < 256; s++)
            if (len[s] == l) syms[n++] = rotate_symbol(uint8_t(s));
        if (count[l] && !lh.min_len) lh.min_len = l;
        if (count[l]) lh.max_len = l;
    }
    lh.n_syms = uint32_t(n);
    uint64_t* lj_end = reinterpret_cast<uint64_t*>(blob + kLutOffLjEnd);
    uint32_t* delta = reinterpret_cast<uint32_t*>(blob + kLutOffDelta);
    lj_end[0] = 0;
    for (int l = 1; l <= 32; l++) {
        lj_end[l] = (first[l] + count[l]) << (32 - l);
        delta[l] = base[l] - uint32_t(first[l]);  // wraps; used modulo 2^32
    }

    // the code at the front of every 12-bit value, when it has at most 12
    // bits: front[v] = length << 8 | rotated symbol, 0 if longer (canonical
    // codes are ranges of consecutive values, so each fills its range)
    static_assert(kPeekBits == 12, "front table covers the widest level-1 table");
    uint16_t front[1u << kPeekBits] = {0};
    {
        int idx = 0;
        for (int l = 1; l <= kPeekBits; l++) {
            for (uint64_t j = 0; j < count[l]; j++, idx++) {
                const uint32_t lo = uint32_t((first[l] + j) << (kPeekBits - l));
                const uint32_t hi = lo + (1u << (kPeekBits - l));
                for (uint32_t v = lo; v < hi; v++) front[v] = uint16_t((l << 8) | syms[idx]);
            }
        }
    }

    // level 1 for a K-bit peek: walk the complete codes at the front of every
    // K-bit value; the count table only exists for K = 12
    auto level1 = [&](int K, uint32_t* ctab, uint16_t* mtab, uint32_t* dtab) {
        for (uint32_t v = 0; v < (1u << K); v++) {
            uint32_t mask = 0, count = 0, syms4 = 0, n4 = 0, used4 = 0;
            int pos = 0;
            while (pos < K) {
                // the bits of v from pos on, at the front of 12 bits (zeros after)
                const uint32_t f = front[(v << (kPeekBits - K + pos)) & ((1u << kPeekBits) - 1)];
                const int l = int(f >> 8);
                if (l == 0 || pos + l > K) break;
                mask |= 1u << pos;
                count++;
                if (n4 < kDecodeSyms) {
                    syms4 |= uint32_t(f & 0xFFu) << (8 * n4);
                    n4++;
                    used4 = uint32_t(pos + l);
                }
                pos += l;
            }
            if (ctab) ctab[v] = count ? ((uint32_t(pos) << 16) | count) : (kEscape << 16);
            mtab[v] = uint16_t(mask);
            dtab[2 * v] = n4 ? syms4 : 0u;
            dtab[2 * v + 1] = n4 ? ((used4 << 16) | (8 * n4)) : (kEscape << 16);
        }
    };
    // level 2 for codes longer than K: up to kLongBits bits by their 20-bit
    // prefix, from the first code longer than K on; none (count 0) when the
    // long codes need more than `cap` prefixes.  A code of l bits covers
    // 2^(20 - l) consecutive prefixes.
    auto level2 = [&](int K, uint16_t* ltab, uint32_t cap, uint32_t* long_base, uint32_t* long_count) {
        const uint64_t region = (uint64_t(1) << 32) - lj_end[K];  // code space of long codes
        const uint64_t n_long = (region + (uint64_t(1) << (32 - kLongBits)) - 1) >> (32 - kLongBits);
        *long_base = uint32_t(lj_end[K] >> (32 - kLongBits));
        *long_count = (lj_end[K] < (uint64_t(1) << 32) && n_long <= cap) ? uint32_t(n_long) : 0u;
        if (!*long_count) return;
        for (int l = K + 1; l <= int(kLongBits); l++) {
            for (uint64_t j = 0; j < count[l]; j++) {
                const uint64_t lo = (first[l] + j) << (kLongBits - l);
                const uint64_t hi = lo + (uint64_t(1) << (kLongBits - l));
                const uint16_t e = uint16_t(syms[base[l] + j] | (uint32_t(l) << 8));
                for (uint64_t v = lo; v < hi; v++) ltab[v - *long_base] = e;
            }
        }
    };
    level1(kPeekBits, reinterpret_cast<uint32_t*>(blob + kLutOffCount), reinterpret_cast<uint16_t*>(blob + kLutOffMask),
           reinterpret_cast<uint32_t*>(blob + kLutOffDecode));
    level2(kPeekBits, reinterpret_cast<uint16_t*>(blob + kLutOffLong), kLongEntries, &lh.long_base, &lh.long_count);
    for (int K = 10; K >= 8; K--) {
        uint8_t* sec = blob + narrow_off(K);
        level1(K, nullptr, reinterpret_cast<uint16_t*>(sec + narrow_mask_off(K)),
               reinterpret_cast<uint32_t*>(sec + narrow_decode_off(K)));
        level2(K, reinterpret_cast<uint16_t*>(sec + narrow_long_off(K)), narrow_long_entries(K),
               &lh.narrow_long[narrow_index(K)][0], &lh.narrow_long[narrow_index(K)][1]);
    }
    std::memcpy(blob, &lh, sizeof(lh));
    return DF11_OK;
}

df11_status df11_compress_workspace_size(uint64_t n_elems, uint64_t* bytes) {
    if (!bytes) return fail(DF11_ERR_INVALID, "df11_compress_workspace_size: null pointer");
    const uint64_t chunks = (n_elems + kEncChunk - 1) / kEncChunk;
    *bytes = ws_bytes(chunks);
    return DF11_OK;
}

}  // extern "C"
