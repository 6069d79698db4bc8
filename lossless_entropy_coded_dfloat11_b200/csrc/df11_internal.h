// Internal declarations shared by the library's host and device code.
// Not part of the C ABI.
#pragma once

#include <cstdint>

#include "../../include/df11.h"

namespace df11 {

// ---------------------------------------------------------------------------
// Decode tables ("Decodificacao com LUT hierarquica" in the DFloat11 summary:
// lookup tables small enough for on-chip memory instead of a bit-level tree
// walk).  Two levels:
//
//   level 1, indexed by the next K stream bits
//     count table  (K = kCountBits):  uint16 = start mask | consumed << 12.
//         Bit j of the 12-bit mask is set when a complete code starts at
//         offset j of the peek; `consumed` is the number of bits the complete
//         codes use.  0 = the first code is longer than K bits.
//     decode table (K = kDecodeBits): uint32 = up to three symbols (bits
//         0..23, first symbol lowest) | n << 24 | consumed << 26.
//         n = number of complete codes decoded (<= 3); 0 = first code longer
//         than K bits.
//   level 2, for codes longer than K: canonical codes of one length are
//     consecutive integers, so a code's length is the smallest l with
//     peek32 < lj_end[l] (lj_end[l] = end of the length-l codes, shifted to
//     the top of 32 bits), and its symbol is syms[(peek32 >> (32 - l)) +
//     delta[l]] with syms sorted by (length, value).
//
// The pages cut the tree into 8-bit-high subtrees with 256-entry tables and
// re-use exponent values 240..255 as pointers; here every exponent value
// must stay representable, so level 2 is the comparison ladder instead.
// ---------------------------------------------------------------------------
constexpr uint32_t kLutMagic = 0x31314644u;  // "DF11"
constexpr int kCountBits = 12;
constexpr int kDecodeBits = 12;

struct LutHeader {
    uint32_t magic;
    uint32_t count_bits;
    uint32_t decode_bits;
    uint32_t n_syms;
    uint32_t min_len;
    uint32_t max_len;
    uint32_t pad[10];
};
static_assert(sizeof(LutHeader) == 64, "LutHeader is 64 bytes");

constexpr uint64_t align16(uint64_t v) { return (v + 15) & ~uint64_t(15); }
constexpr uint64_t kLutOffLjEnd = 64;                                       // uint64[33]
constexpr uint64_t kLutOffDelta = align16(kLutOffLjEnd + 33 * 8);           // uint32[33]
constexpr uint64_t kLutOffSyms = align16(kLutOffDelta + 33 * 4);            // uint8[256]
constexpr uint64_t kLutOffCount = align16(kLutOffSyms + 256);               // uint16[2^K]
constexpr uint64_t kLutOffDecode = align16(kLutOffCount + (2ull << kCountBits));  // uint32[2^K]
constexpr uint64_t kLutBytes = align16(kLutOffDecode + (4ull << kDecodeBits));

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

}  // namespace df11
