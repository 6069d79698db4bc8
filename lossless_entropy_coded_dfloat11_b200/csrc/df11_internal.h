// Internal declarations shared by the library's host and device code.
// Not part of the C ABI.
#pragma once

#include <cstdint>

#include "../../include/df11.h"

namespace df11 {

// ---------------------------------------------------------------------------
// Decode tables ("Decodificacao com LUT hierarquica" in the DFloat11 summary:
// lookup tables small enough for on-chip memory instead of a bit-level tree
// walk).  Two levels.
//
// Level 1 is indexed by the next K = 12 stream bits:
//   count table  uint32 = consumed << 16 | count
//       count    = complete codes at the front of the peek (0..12)
//       consumed = bits those codes use (1..12)
//       The kernel keeps (bit position << 16 | code count) in one register,
//       so one add advances both.
//   mask table   uint16, bit j set when a complete code starts at offset j
//       (used once per window, to drop codes that start past its end).
//   decode table uint2: x = up to four symbols (first in bits 0..7, unused
//       bytes zero), each an exponent rotated right by one bit (bit 0 moved
//       to bit 7) so that the merge needs only bit-selects;
//       y = consumed << 16 | 8n, n = codes decoded (1..4).  The kernels keep
//       (bit position << 16 | 8 x bytes produced) in one register, whose
//       low five bits then are the shift that places the next symbols.
//   A peek whose first code is longer than K bits (or matches no code) holds
//   the escape value kEscape << 16 (count 0, n 0, symbols 0): adding it
//   pushes the bit position past every window end, so the fast loops need
//   no escape test; the slow path undoes it.
// Level 2, for codes longer than K.  Canonical codes put every code longer
//   than K bits at the top of the code space, from lj_end[K] up (lj_end[l] =
//   end of the codes of length <= l, shifted to the top of 32 bits).
//   * long table uint16[<= 4096]: entry i describes the 20-bit prefix
//     (lj_end[K] >> 12) + i: rotated symbol | length << 8 when the code has
//     at most 20 bits, else 0.  Built only when the long codes fit in 4096
//     such prefixes (LutHeader::long_count, 0 otherwise).
//   * ladder: a code's length is the smallest l with peek32 < lj_end[l], its
//     symbol syms[(peek32 >> (32 - l)) + delta[l]] with syms sorted by
//     (length, value) (stored rotated, as above).
//
// The pages cut the tree into 8-bit-high subtrees with 256-entry tables and
// re-use exponent values 240..255 as pointers; here every exponent value
// must stay representable, so level 2 is the comparison ladder instead.
// ---------------------------------------------------------------------------
constexpr uint32_t kLutMagic = 0x31314644u;  // "DF11"
constexpr int kPeekBits = 12;
constexpr uint32_t kEscape = 512;            // > any bit position a thread decodes (<= 256) + K
constexpr uint32_t kDecodeSyms = 4;          // symbols per decode-table entry

struct LutHeader {
    uint32_t magic;
    uint32_t peek_bits;
    uint32_t escape;
    uint32_t n_syms;
    uint32_t min_len;
    uint32_t max_len;
    uint32_t long_base;   // (lj_end[K] >> 12): 20-bit prefix of the first long code
    uint32_t long_count;  // entries of the long table, 0 = ladder only
    uint32_t narrow_long[3][2];  // long_base, long_count of the narrow sections (K = 10, 9, 8)
    uint32_t pad[2];
};
static_assert(sizeof(LutHeader) == 64, "LutHeader is 64 bytes");

constexpr uint64_t align16(uint64_t v) { return (v + 15) & ~uint64_t(15); }
constexpr uint64_t kLutEntries = uint64_t(1) << kPeekBits;
constexpr uint64_t kLutOffLjEnd = 64;                                       // uint64[33]
constexpr uint64_t kLutOffDelta = align16(kLutOffLjEnd + 33 * 8);           // uint32[33]
constexpr uint64_t kLutOffSyms = align16(kLutOffDelta + 33 * 4);            // uint8[256]
constexpr uint64_t kLutOffCount = align16(kLutOffSyms + 256);               // uint32[2^K]
constexpr uint64_t kLutOffMask = align16(kLutOffCount + 4 * kLutEntries);   // uint16[2^K]
constexpr uint64_t kLutOffDecode = align16(kLutOffMask + 2 * kLutEntries);  // uint2[2^K]
constexpr uint32_t kLongEntries = 4096;
constexpr uint32_t kLongBits = 20;                                          // long-table resolution
constexpr uint64_t kLutOffLong = align16(kLutOffDecode + 8 * kLutEntries);  // uint16[kLongEntries]

// Narrow level-1 sections: the same mask and decode tables for a K-bit peek,
// K = 10, 9 or 8 (the pages' 256-entry first level), each with its own long
// table for the codes longer than K.  A table of 2^K entries is small enough
// to be staged in shared memory once per 8-byte bank pair (16 copies, copy c
// in bank pair c), so the 16 lanes of a half-warp always read distinct bank
// pairs: one wavefront per half-warp, whatever the indices.
//   section(K) = mask u16[2^K] | long u16[narrow_long_entries(K)] | decode uint2[2^K]
constexpr uint32_t narrow_long_entries(int K) { return K == 8 ? 8192u : 4096u; }
constexpr uint64_t narrow_mask_off(int) { return 0; }
constexpr uint64_t narrow_long_off(int K) { return uint64_t(2) << K; }
constexpr uint64_t narrow_decode_off(int K) { return narrow_long_off(K) + 2 * uint64_t(narrow_long_entries(K)); }
constexpr uint64_t narrow_bytes(int K) { return align16(narrow_decode_off(K) + (uint64_t(8) << K)); }
constexpr int narrow_index(int K) { return 10 - K; }  // LutHeader::narrow_long row
constexpr uint64_t kLutOffNarrow = align16(kLutOffLong + 2 * kLongEntries);
constexpr uint64_t narrow_off(int K) {
    return K == 10 ? kLutOffNarrow : K == 9 ? kLutOffNarrow + narrow_bytes(10)
                                            : kLutOffNarrow + narrow_bytes(10) + narrow_bytes(9);
}
constexpr uint64_t kLutBytes = narrow_off(8) + narrow_bytes(8);

// Canonical code per value (DEFLATE-style construction); false if the
// lengths overflow the code space.
bool canonical_codes(const uint8_t* len, uint32_t* code);

// Sizes of the container arrays for a header whose n_elems, total_bits and
// threads_per_block are set.
void fill_sizes(df11_header* h);

// Set this thread's error message; returns `st` for chaining.
df11_status fail(df11_status st, const char* fmt, ...);

// Kernel-side limits
constexpr uint32_t kEncChunk = 4096;       // elements per bit-pack CTA
constexpr uint32_t kEncThreads = 256;      // threads per bit-pack CTA
constexpr uint32_t kEncPerThread = kEncChunk / kEncThreads;
// At most this many CTAs (chunk ranges) in an encode grid; the workspace holds
// one 256-entry histogram per range.
constexpr uint32_t kMaxEncRanges = 2048;
// Workspace layout of the compress entry points, in bytes: the global
// histogram (256 x u64), the range tag, the look-back descriptors, chunk
// ticket and abort flag (8 (chunks + 2)), then the per-range histograms
// (256 x u32 each).
constexpr uint64_t kWsTagOff = 2048;
constexpr uint64_t kWsDescOff = kWsTagOff + 64;
inline uint64_t ws_range_hist_off(uint64_t chunks) { return kWsDescOff + ((8 * (chunks + 2) + 15) & ~uint64_t(15)); }
inline uint64_t ws_bytes(uint64_t chunks) {
    const uint64_t ranges = chunks < kMaxEncRanges ? chunks : kMaxEncRanges;
    return ws_range_hist_off(chunks) + 1024 * ranges + 64;
}
// Independent-chunk variant of the container: one 32-bit start bit per
// kIndChunk elements replaces Gaps and block offsets.
constexpr uint32_t kIndChunk = 64;
static_assert(kIndChunk % kEncPerThread == 0, "chunk starts fall on encode-thread boundaries");

}  // namespace df11
