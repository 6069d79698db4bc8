// DF11 decompression kernels for sm_100a.
//
// Follows the two-phase design of "DFloat11: compressao sem perda para
// inferencia em GPU que reduz LLMs para 70% do tamanho", section "Kernel de
// GPU em 2 etapas e metadados auxiliares": every thread owns one 8-byte
// window of EncodedExponent and decodes the codes that start in it, beginning
// at its 5-bit gap; phase 1 counts them, a prefix sum over the thread block
// turns counts into output positions (added to the block's stored position),
// and phase 2 decodes again into an on-chip buffer that is written to HBM
// with coalesced stores.  One launch covers a whole stream, i.e. every matrix
// of a transformer block ("Descompressao por bloco de transformer").
//
// B200 specifics:
//   * persistent grid: the decode tables are copied to shared memory once
//     per CTA and serve every thread block of the stream;
//   * thread blocks of T = 32 or 64 threads are decoded by one warp each,
//     with no CTA barrier at all: the prefix sum is five shuffles and the
//     staging buffer is the warp's own; for T = 64 each lane decodes its two
//     windows as one 128-bit run from the first window's gap (the second
//     window's codes are the ones the run reaches); larger T use a
//     block-wide scan;
//   * software pipelining: the next block's window, gap and output positions
//     are loaded while the current one is decoded, and the current block's
//     sign+mantissa bytes are requested before its decode starts;
//   * the decode loops keep (bit position << 16 | counter) in one register
//     and advance both with one add; one loop runs per 32 bits of the run so
//     each peek is one funnel shift of a word pair; codes
//     longer than the 12-bit tables leave through an escape value that pushes
//     the bit position out of the window, so the fast loops have one test;
//   * symbols are gathered in a register pair and leave as aligned 32-bit
//     words; a thread's first word, shared with the previous thread, is
//     written byte-wise after a barrier.  The warp kernel decodes each
//     window only once, into a per-thread shared-memory slot, and copies the
//     slot into place after the scan; the block kernel decodes twice (count,
//     then decode into place);
//   * exponents are staged rotated right by one bit, so the merge is two
//     bit-selects and two byte-permutes per four elements.  The warp kernel
//     merges 8-element units (8-byte shared load, 8-byte streaming load, one
//     16-byte streaming store; one store instruction of a warp covers 512
//     contiguous bytes), the block kernel 16-element chunks.
// Indices are 32-bit: n_elems < 2^32 and codes of at most 32 bits keep the
// window count below 2^31.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdio>
#include <cstring>

#include "df11_internal.h"

namespace df11 {
namespace {

struct DecodeArgs {
    const uint8_t* exp;
    const uint4* sm;
    const uint32_t* gaps;
    const uint32_t* off;
    const uint4* lut;
    uint16_t* out;        // BF16 output (streams of BF16 weights)
    uint8_t* out8;        // symbol output (streams of 8-bit symbols)
    uint32_t* status;
    uint32_t n_elems;
    uint32_t n_threads;
    uint32_t block0;     // first thread block to decode
    uint32_t n_blocks;   // thread blocks to decode, from block0
    uint32_t last_wend;  // bits of the last window inside the stream, 1..64
    uint32_t early;      // stage the tables and first loads before waiting for the prior grid
};

struct Tables {
    const uint32_t* ctab;             // count table
    const uint16_t* mtab;             // start-mask table
    const uint2* dtab;                // decode table
    const unsigned long long* lj_end; // level 2
    const uint32_t* delta;
    const uint8_t* syms;
};

__device__ __forceinline__ Tables tables_at(const uint8_t* s_lut) {
    Tables t;
    t.ctab = reinterpret_cast<const uint32_t*>(s_lut + kLutOffCount);
    t.mtab = reinterpret_cast<const uint16_t*>(s_lut + kLutOffMask);
    t.dtab = reinterpret_cast<const uint2*>(s_lut + kLutOffDecode);
    t.lj_end = reinterpret_cast<const unsigned long long*>(s_lut + kLutOffLjEnd);
    t.delta = reinterpret_cast<const uint32_t*>(s_lut + kLutOffDelta);
    t.syms = s_lut + kLutOffSyms;
    return t;
}

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

// 32 stream bits starting at bit `pos` (0 <= pos < 64) of the 96-bit window
// w0:w1:w2 (MSB first).
__device__ __forceinline__ uint32_t peek32(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t pos) {
    const uint32_t hi = pos < 32 ? w0 : w1;
    const uint32_t lo = pos < 32 ? w1 : w2;
    return __funnelshift_l(lo, hi, pos);
}

// Level 2: length of the canonical code at the top of `peek`, 0 if none.
// Codes shorter than `from` bits are known not to match.
__device__ __forceinline__ int code_length(const unsigned long long* lj_end, uint32_t peek, int from) {
    for (int l = from; l <= 32; l++)
        if ((unsigned long long)peek < lj_end[l]) return l;
    return 0;
}

__device__ __forceinline__ uint32_t code_symbol(const Tables& t, uint32_t peek, int l) {
    return t.syms[((peek >> (32 - l)) + t.delta[l]) & 0xFFu];
}

// Raw loads of one thread's window, issued early and finished later.
struct RawWindow {
    uint2 v;        // the 8-byte window
    uint32_t v2;    // 4-byte lookahead
    uint32_t glo, ghi;
};

struct Window {
    uint32_t w0, w1, w2;  // 96 stream bits, MSB first
    uint32_t start;       // first code start in the window (the gap)
    uint32_t wend;        // end of the window inside the stream, 0..64
};

// tg = window index; its gap field sits in gap words gword, gword + 1.
__device__ __forceinline__ RawWindow load_window(const DecodeArgs& a, uint32_t tg, uint32_t gword) {
    RawWindow r;
    if (tg < a.n_threads) {
        const uint8_t* base = a.exp + 8 * size_t(tg);
        r.v = __ldg(reinterpret_cast<const uint2*>(base));
        r.v2 = __ldg(reinterpret_cast<const uint32_t*>(base + 8));
        const uint32_t* gp = a.gaps + gword;
        r.glo = __ldg(gp);
        r.ghi = __ldg(gp + 1);
    } else {
        r.v = make_uint2(0, 0);
        r.v2 = r.glo = r.ghi = 0;
    }
    return r;
}

__device__ __forceinline__ Window finish_window(const DecodeArgs& a, const RawWindow& r, uint32_t tg,
                                                uint32_t gshift) {
    Window w;
    w.w0 = bswap32(r.v.x);
    w.w1 = bswap32(r.v.y);
    w.w2 = bswap32(r.v2);
    w.start = __funnelshift_r(r.glo, r.ghi, gshift) & 31u;
    const uint32_t last = a.n_threads - 1;
    w.wend = tg < last ? 64u : (tg == last ? a.last_wend : 0u);
    return w;
}

// Phase 1: number of codes that start in [start, wend).  Sets `bad` if a
// bit pattern matches no code (corrupt stream).
__device__ __forceinline__ uint32_t count_codes(const Window& w, const Tables& t, bool& bad) {
    const uint32_t lim1 = min(w.wend, 32u) << 16;
    const uint32_t lim2 = w.wend << 16;
    uint32_t acc = w.start << 16;  // bit position << 16 | codes counted
    uint32_t e = 0, idx = 0;
    for (;;) {
        while (acc < lim1) {
            idx = __funnelshift_l(w.w1, w.w0, acc >> 16) >> (32 - kPeekBits);
            e = t.ctab[idx];
            acc += e;
        }
        while (acc < lim2) {
            idx = __funnelshift_l(w.w2, w.w1, acc >> 16) >> (32 - kPeekBits);
            e = t.ctab[idx];
            acc += e;
        }
        if (acc < (kEscape << 16)) break;
        // a code longer than the table: undo the escape, take it from level 2
        acc -= kEscape << 16;
        const int l = code_length(t.lj_end, peek32(w.w0, w.w1, w.w2, acc >> 16), kPeekBits + 1);
        if (!l) {
            bad = true;
            return 0;
        }
        acc += (uint32_t(l) << 16) | 1u;
        e = 0;
    }
    uint32_t cnt = acc & 0xFFFFu;
    if (e) {  // the last table step may hold codes starting at or past wend
        const uint32_t s = w.wend - ((acc >> 16) - (e >> 16));
        if (s < uint32_t(kPeekBits)) cnt -= __popc(uint32_t(t.mtab[idx]) >> s);
    }
    return cnt;
}

// Phase 2: decode the same codes into staging bytes [pos0, pos0 + cnt).
// Symbols collect in a register pair and leave as aligned 32-bit words.  The
// thread's first word is not stored when it starts mid-word (it is shared
// with the previous thread): it is returned, for write_head after a barrier.
// A stored word holding the thread's last symbols may carry up to three
// bytes decoded past the window end; those positions are head bytes of the
// following threads (which start mid-word) and are rewritten by them.
__device__ __forceinline__ uint32_t decode_codes(const Window& w, const Tables& t, uint32_t* stage32,
                                                 uint32_t pos0, uint32_t cnt) {
    if (cnt == 0) return 0;
    const uint32_t lim1 = min(w.wend, 32u) << 16;
    const uint32_t lim2 = w.wend << 16;
    const uint32_t last_word = (pos0 + cnt - 1) >> 2;
    const uint32_t skip_word = (pos0 & 3u) ? (pos0 >> 2) : 0xFFFFFFFFu;
    uint32_t wi = pos0 >> 2;  // word the pending bytes belong to
    uint32_t lo = 0, head = 0;
    // bit position << 16 | 8 x bytes pending: the low five bits are the shift
    // that places the next symbols in `lo`
    uint32_t acc = (w.start << 16) | ((pos0 & 3u) << 3);
    auto put = [&](uint32_t x, uint32_t y) {
        lo |= __funnelshift_l(0u, x, acc);                // x << (acc & 31)
        const uint32_t hi = __funnelshift_l(x, 0u, acc);  // bytes spilling past lo
        acc += y;
        if (acc & 32u) {  // a word is complete
            if (wi != skip_word) stage32[wi] = lo; else head = lo;
            wi++;
            lo = hi;
            acc -= 32u;
        }
    };
    for (;;) {
        while (acc < lim1) {
            const uint2 e = t.dtab[__funnelshift_l(w.w1, w.w0, acc >> 16) >> (32 - kPeekBits)];
            put(e.x, e.y);
        }
        while (acc < lim2) {
            const uint2 e = t.dtab[__funnelshift_l(w.w2, w.w1, acc >> 16) >> (32 - kPeekBits)];
            put(e.x, e.y);
        }
        if (acc < (kEscape << 16)) break;
        acc -= kEscape << 16;
        const uint32_t pk = peek32(w.w0, w.w1, w.w2, acc >> 16);
        int l = code_length(t.lj_end, pk, kPeekBits + 1);
        l = l ? l : 1;
        put(code_symbol(t, pk, l), (uint32_t(l) << 16) | 8u);
    }
    if (acc & 31u) {
        if (wi == skip_word) head = lo;
        else if (wi <= last_word) stage32[wi] = lo;
    }
    return head;
}

// After a barrier: the bytes of this thread's first word when it starts
// mid-word, from the word phase 2 kept back.
__device__ __forceinline__ void write_head(uint8_t* stage, uint32_t pos0, uint32_t cnt, uint32_t head) {
    const uint32_t b0 = pos0 & 3u;
    const uint32_t room = (4u - b0) & 3u;
    const uint32_t k = cnt < room ? cnt : room;
    uint8_t* d = stage + pos0;
    if (k > 0) d[0] = uint8_t(head >> (8 * b0));
    if (k > 1) d[1] = uint8_t(head >> (8 * b0 + 8));
    if (k > 2) d[2] = uint8_t(head >> 24);
}

// Four BF16 values from four staged (rotated) exponent bytes r4 and four
// sign+mantissa bytes s4: the high output byte is sign | e >> 1 and the low
// one (e & 1) << 7 | mantissa, i.e. two bit-selects between r4 and s4.
__device__ __forceinline__ void merge4(uint32_t r4, uint32_t s4, uint32_t& o01, uint32_t& o23) {
    const uint32_t hi = (s4 & 0x80808080u) | (r4 & 0x7F7F7F7Fu);
    const uint32_t lo = (r4 & 0x80808080u) | (s4 & 0x7F7F7F7Fu);
    o01 = __byte_perm(lo, hi, 0x5140);
    o23 = __byte_perm(lo, hi, 0x7362);
}

// Merge and store chunk c (elements 16c..16c+15) of the range [lo, hi).
__device__ __forceinline__ void merge_chunk(const uint4 ev, const uint4 sv, uint32_t c, uint32_t lo, uint32_t hi,
                                            uint16_t* __restrict__ out) {
    uint4 o0, o1;
    merge4(ev.x, sv.x, o0.x, o0.y);
    merge4(ev.y, sv.y, o0.z, o0.w);
    merge4(ev.z, sv.z, o1.x, o1.y);
    merge4(ev.w, sv.w, o1.z, o1.w);
    uint4* dst = reinterpret_cast<uint4*>(out) + 2 * size_t(c);
    const uint32_t i0 = 16 * c;
    if (i0 >= lo && i0 + 16 <= hi) {
        __stcs(dst, o0);
        __stcs(dst + 1, o1);
    } else {
        const uint32_t words[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
        uint16_t* d16 = reinterpret_cast<uint16_t*>(dst);
#pragma unroll
        for (int k = 0; k < 16; k++) {
            const uint32_t i = i0 + k;
            if (i >= lo && i < hi) d16[k] = uint16_t(words[k >> 1] >> (16 * (k & 1)));
        }
    }
}

// Merge 8 elements and store them as one 16-byte streaming store: staged
// (rotated) exponents at shared address ev_s + EV_OFF, sign+mantissa bytes
// sv, destination dst + DST_OFF bytes; m = 0x80808080.  A warp storing
// units 32 apart per instruction writes 512 contiguous bytes.
template <int EV_OFF = 0, int DST_OFF = 0>
__device__ __forceinline__ void merge_store8(uint32_t ev_s, const uint2 sv, uint4* dst, uint32_t m) {
    asm volatile(
        "{\n\t"
        ".reg .b32 e0, e1, h, l, o0, o1, o2, o3;\n\t"
        "ld.shared.v2.u32 {e0, e1}, [%0+%5];\n\t"
        "lop3.b32 h, %1, e0, %4, 0xE4;\n\t"
        "lop3.b32 l, e0, %1, %4, 0xE4;\n\t"
        "prmt.b32 o0, l, h, 0x5140;\n\t"
        "prmt.b32 o1, l, h, 0x7362;\n\t"
        "lop3.b32 h, %2, e1, %4, 0xE4;\n\t"
        "lop3.b32 l, e1, %2, %4, 0xE4;\n\t"
        "prmt.b32 o2, l, h, 0x5140;\n\t"
        "prmt.b32 o3, l, h, 0x7362;\n\t"
        "st.global.cs.v4.u32 [%3+%6], {o0, o1, o2, o3};\n\t"
        "}"
        :
        : "r"(ev_s), "r"(sv.x), "r"(sv.y), "l"(dst), "r"(m), "n"(EV_OFF), "n"(DST_OFF)
        : "memory");
}

// Merge and store unit u (elements 8u..8u+7) of the range [lo, hi).
__device__ __forceinline__ void merge_unit(const uint2 ev, const uint2 sv, uint32_t u, uint32_t lo, uint32_t hi,
                                           uint16_t* __restrict__ out) {
    uint4 o;
    merge4(ev.x, sv.x, o.x, o.y);
    merge4(ev.y, sv.y, o.z, o.w);
    uint4* dst = reinterpret_cast<uint4*>(out) + size_t(u);
    const uint32_t i0 = 8 * u;
    if (i0 >= lo && i0 + 8 <= hi) {
        __stcs(dst, o);
    } else {
        const uint32_t words[4] = {o.x, o.y, o.z, o.w};
        uint16_t* d16 = reinterpret_cast<uint16_t*>(dst);
#pragma unroll
        for (int k = 0; k < 8; k++) {
            const uint32_t i = i0 + k;
            if (i >= lo && i < hi) d16[k] = uint16_t(words[k >> 1] >> (16 * (k & 1)));
        }
    }
}

// Sixteen staged symbols rotated back: the tables hold each symbol rotated
// right by one bit (for the BF16 merge); an 8-bit symbol is its byte rotated
// left by one.
__device__ __forceinline__ uint4 unrotate16(const uint4 r) {
    auto rol1 = [](uint32_t w) { return ((w << 1) & 0xFEFEFEFEu) | ((w >> 7) & 0x01010101u); };
    return make_uint4(rol1(r.x), rol1(r.y), rol1(r.z), rol1(r.w));
}

// the K = 12 tables: everything before the narrow sections
constexpr uint64_t kLutWideBytes = kLutOffNarrow;


__device__ __forceinline__ bool block_consistent(uint32_t off0, uint32_t off1, uint32_t total, uint32_t n) {
    return off0 <= off1 && off1 <= n && total == off1 - off0;
}

// ---------------------------------------------------------------------------
// Table staging through the bulk-copy engine: one thread initialises an
// mbarrier, announces the bytes and issues one cp.async.bulk per piece; the
// copies then run without any thread's registers, whatever the CTA size (a
// CTA of a few warps would otherwise need many dependent load rounds).  The
// issuing thread waits on the mbarrier -- a bounded wait -- and a CTA barrier
// passes the tables on.  A wait that runs out (never expected) waits once
// more for the copies in flight, then the CTA reports the stream corrupt and
// stops.
// ---------------------------------------------------------------------------
constexpr uint32_t kBulkWaitLimit = 1u << 20;

__device__ __forceinline__ void bulk_begin(uint32_t bar, uint32_t tx_bytes) {
    asm volatile(
        "mbarrier.init.shared::cta.b64 [%0], 1;\n\t"
        "fence.mbarrier_init.release.cluster;\n\t"
        "fence.proxy.async.shared::cta;\n\t"
        "mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
        ::"r"(bar), "r"(tx_bytes) : "memory");
}

// bytes: a multiple of 16; both addresses 16-byte aligned
__device__ __forceinline__ void bulk_copy(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

__device__ __forceinline__ bool bulk_wait(uint32_t bar) {
    for (uint32_t i = 0; i < kBulkWaitLimit; i++) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done) : "r"(bar) : "memory");
        if (done) return true;
    }
    return false;
}

// Thread 0: wait for the staged tables; false (after a second bounded wait
// for the copies still in flight) if they never arrived.
__device__ __forceinline__ bool bulk_end(uint32_t bar) {
    if (bulk_wait(bar)) return true;
    bulk_wait(bar);
    return false;
}

// Kernels launched with programmatic stream serialisation start while the
// previous kernel on the stream drains; nothing is read before this.
__device__ __forceinline__ void wait_for_prior_grids() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_next_grid() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// After the table copy and a CTA barrier: false (and the stream reported
// corrupt) when the staged tables do not carry the library's magic word -- a
// table buffer never filled, or the tables of a stream whose encode gave up.
__device__ __forceinline__ bool tables_valid(const uint8_t* s_lut, uint32_t* status) {
    if (reinterpret_cast<const LutHeader*>(s_lut)->magic == kLutMagic) return true;
    if (threadIdx.x == 0 && status) atomicOr(status, uint32_t(DF11_ERR_CORRUPT));
    return false;
}

// ---------------------------------------------------------------------------
// T = 32 and T = 64: one warp decodes one thread block at a time, each lane
// WPL = T / 32 consecutive windows; no CTA barrier after the table copy.
//
// Decode once: each thread decodes its windows a single time into a private
// slot of shared memory and learns its count from the bytes it wrote,
// corrected for codes of the last table step that start past the run's end.
// After the warp's prefix sum the slots are copied, one aligned word at a
// time, into the block's contiguous staging buffer; the first word of a slot
// range that starts mid-word is written byte-wise after a warp barrier, and a
// last word's bytes past the thread's range belong to such heads, so they are
// overwritten then.  The level-1 count table is not needed here.
//
// The merge works on 8-element units (8 sign+mantissa bytes in, one 16-byte
// store out); lane L takes units L, L + 32, ..., so each store instruction
// of the warp covers 512 contiguous bytes.  Each warp takes a contiguous run
// of thread blocks, so the unit that straddles two consecutive blocks is
// stored once, as a whole, by the later block: the earlier block leaves it
// in the staging buffer and the warp carries its bytes over; only the first
// and last unit of a run need element-wise stores.
// ---------------------------------------------------------------------------
// Per-warp buffers depend on the shortest code length and the windows per
// lane: a lane's 64 WPL bits hold at most 64 WPL / min_len code starts, plus
// up to three symbols decoded past their end.  The slots are stored transposed (word k of lane L at word
// 32k + L), so each lane always uses the same bank: the decode loop's
// stores, which happen at a different word offset in every lane, and the
// copy's loads are free of bank conflicts.
template <int MIN_LEN, int WPL>
struct WarpLayout {
    static constexpr uint32_t kMaxCodes = 64 * WPL / MIN_LEN;
    static constexpr uint32_t kSlotWords = (kMaxCodes + 3 + 3) / 4;
    static constexpr uint32_t kSlots = 32 * kSlotWords * 4;
    static constexpr uint32_t kStage = 32 * kMaxCodes + 64;  // + head (15) + spill, rounded
    static constexpr uint32_t kBytes = kSlots + kStage;
};
// shared-memory copy of the tables this kernel uses: ladder, deltas and
// symbols, then the mask, decode and long tables
constexpr uint32_t kCompactSmall = uint32_t(kLutOffCount);
constexpr uint32_t kCompactMask = kCompactSmall;
constexpr uint32_t kCompactDecode = kCompactMask + uint32_t(kLutOffDecode - kLutOffMask);
constexpr uint32_t kCompactLong = kCompactDecode + uint32_t(kLutOffLong - kLutOffDecode);
constexpr uint32_t kCompactBytes = kCompactDecode + uint32_t(kLutWideBytes - kLutOffDecode);


// Shared-memory layout of the tables a warp kernel decodes with.  K = 12: the
// compact copy above, decode table in one copy (8-byte entries at random
// 12-bit indices: ~5 wavefronts per warp lookup).  K < 12: a narrow section,
// its decode table stored once per 8-byte bank pair -- entry i of copy c at
// 8-byte slot 16 i + c, lane L reading copy L % 16 -- so every lookup takes
// one wavefront per half-warp.
template <int K>
struct TableLayout {
    static constexpr bool kNarrow = K != kPeekBits;
    static constexpr uint32_t kRep = kNarrow ? 16u : 1u;  // copies of the decode table
    static constexpr uint32_t kStride = 8 * kRep;          // bytes between entries
    static constexpr uint32_t kMask = kNarrow ? kCompactSmall : kCompactMask;
    static constexpr uint32_t kLong = kNarrow ? kMask + (2u << K) : kCompactLong;
    static constexpr uint32_t kLongEnd = kNarrow ? kLong + 2 * narrow_long_entries(K) : kCompactBytes;
    static constexpr uint32_t kDecode = kNarrow ? (kLongEnd + 127) & ~127u : kCompactDecode;
    static constexpr uint32_t kBytes = kNarrow ? kDecode + (kRep * 8u << K) : kCompactBytes;
};


// Thread 0: the warp kernel's tables by bulk copies (the small part, then
// the mask and long tables, and for K = 12 the decode table); the narrow
// decode table's 16 copies are written by every thread (copy_narrow_decode).
template <int K>
__device__ __forceinline__ void bulk_warp_tables(uint8_t* s, const uint8_t* g, uint32_t bar) {
    using TL = TableLayout<K>;
    const uint32_t s0 = uint32_t(__cvta_generic_to_shared(s));
    if constexpr (!TL::kNarrow) {
        constexpr uint32_t rest = uint32_t(kLutWideBytes - kLutOffMask);
        bulk_begin(bar, kCompactSmall + rest);
        bulk_copy(s0, g, kCompactSmall, bar);
        bulk_copy(s0 + kCompactMask, g + kLutOffMask, rest, bar);
    } else {
        constexpr uint32_t rest = TL::kLongEnd - TL::kMask;
        bulk_begin(bar, kCompactSmall + rest);
        bulk_copy(s0, g, kCompactSmall, bar);
        bulk_copy(s0 + TL::kMask, g + narrow_off(K), rest, bar);
    }
}

template <int K>
__device__ __forceinline__ void copy_narrow_decode(uint8_t* s, const uint4* g, int nthreads) {
    if constexpr (TableLayout<K>::kNarrow) {
        using TL = TableLayout<K>;
        const uint2* gd = reinterpret_cast<const uint2*>(g) + (narrow_off(K) + narrow_decode_off(K)) / 8;
        uint2* sd = reinterpret_cast<uint2*>(s + TL::kDecode);
        for (int j = threadIdx.x; j < int(TL::kRep << K); j += nthreads) sd[j] = __ldg(gd + (j >> 4));
    }
}

template <int K>
__device__ __forceinline__ void long_table_of(const uint8_t* s, uint32_t& base, uint32_t& count) {
    const LutHeader* h = reinterpret_cast<const LutHeader*>(s);
    if constexpr (TableLayout<K>::kNarrow) {
        base = h->narrow_long[narrow_index(K)][0];
        count = h->narrow_long[narrow_index(K)][1];
    } else {
        base = h->long_base;
        count = h->long_count;
    }
}

// One half of the window (bit positions below lim, peeking at hi:lo) through
// the decode table, in hand-written PTX: 15 instructions per step, with no
// branch but the loop's own.  `acc` is (bit position << 16 | 8 x bytes
// produced so far); its low five bits place the next symbols in `pend`, and a
// word is complete when bit 5 of acc flips.  Every step stores the word under
// construction at `wad` (a shared-window address, stepping 128 bytes in the
// transposed slot), so a completed word is in place when wad moves on;
// `pend` then becomes the spilled bytes through one clamped funnel shift.
// The loop is unrolled twice with acc alternating between two registers.
// The last entry's index and y word stay behind for the end-of-window
// correction.
template <int K, uint32_t STRIDE>
__device__ __forceinline__ void decode_half(uint32_t& acc, uint32_t& pend, uint32_t& wad, uint32_t& idx,
                                            uint32_t& ylast, uint32_t hi, uint32_t lo, uint32_t lim,
                                            uint32_t dtab_s) {
#define DF11_STEP(A, B)                                  \
    "shr.u32 sh, " A ", 16;\n\t"                          \
    "shf.l.wrap.b32 pk, %6, %5, sh;\n\t"                  \
    "shr.u32 %3, pk, %9;\n\t"                             \
    "mad.lo.u32 ad, %3, %10, %8;\n\t"                     \
    "ld.shared.v2.u32 {x, %4}, [ad];\n\t"                 \
    "shf.l.wrap.b32 t1, zero, x, " A ";\n\t"              \
    "or.b32 %1, %1, t1;\n\t"                              \
    "shf.l.wrap.b32 spill, x, zero, " A ";\n\t"           \
    "add.u32 " B ", " A ", %4;\n\t"                       \
    "lop3.b32 t1, " B ", " A ", c32, 0x28;\n\t"           \
    "st.shared.u32 [%2], %1;\n\t"                         \
    "mad.lo.u32 %2, t1, 4, %2;\n\t"                       \
    "shf.r.clamp.b32 %1, %1, spill, t1;\n\t"
    asm volatile(
        "{\n\t"
        ".reg .pred p;\n\t"
        ".reg .u32 sh, pk, ad, x, t1, spill, zero, c32, b;\n\t"
        "mov.u32 zero, 0;\n\t"
        "mov.u32 c32, 32;\n\t"
        "setp.ge.u32 p, %0, %7;\n\t"
        "@p bra DONE;\n\t"
        "LOOP:\n\t"
        DF11_STEP("%0", "b")
        "setp.ge.u32 p, b, %7;\n\t"
        "@p bra DONE_B;\n\t"
        DF11_STEP("b", "%0")
        "setp.lt.u32 p, %0, %7;\n\t"
        "@p bra LOOP;\n\t"
        "bra.uni DONE;\n\t"
        "DONE_B:\n\t"
        "mov.u32 %0, b;\n\t"
        "DONE:\n\t"
        "}"
        : "+r"(acc), "+r"(pend), "+r"(wad), "+r"(idx), "+r"(ylast)
        : "r"(hi), "r"(lo), "r"(lim), "r"(dtab_s), "n"(32 - K), "n"(STRIDE)
        : "memory");
#undef DF11_STEP
}

// The bits one lane of the warp kernel decodes: WPL consecutive 8-byte
// windows read as one run of 64 WPL bits, from the gap of the first window.
// The codes that start in the later windows are exactly the ones the run
// reaches, so their gaps are not needed.
template <int WPL>
struct LaneWindow {
    uint32_t w[2 * WPL + 1];  // 64 WPL stream bits and a 32-bit lookahead, MSB first
    uint32_t start;           // first code start (the first window's gap)
    uint32_t wend;            // end of the run inside the stream, 0..64 WPL
};

template <int WPL>
struct RawLane {
    uint32_t v[2 * WPL];
    uint32_t look;  // lookahead word (WPL = 2: loaded by lane 31 only)
    uint32_t glo, ghi;
};

// tg0 = the lane's first window; its gap field sits in gap words gword, gword + 1.
template <int WPL>
__device__ __forceinline__ RawLane<WPL> load_lane(const DecodeArgs& a, uint32_t tg0, uint32_t gword,
                                                  uint32_t lane) {
    RawLane<WPL> r;
    if (tg0 < a.n_threads) {
        const uint8_t* base = a.exp + 8 * size_t(tg0);
        if constexpr (WPL >= 2) {
#pragma unroll
            for (int h = 0; h < WPL / 2; h++) {
                const uint4 q = __ldg(reinterpret_cast<const uint4*>(base) + h);
                r.v[4 * h] = q.x; r.v[4 * h + 1] = q.y; r.v[4 * h + 2] = q.z; r.v[4 * h + 3] = q.w;
            }
            r.look = lane == 31 ? __ldg(reinterpret_cast<const uint32_t*>(base + 8 * WPL)) : 0u;
        } else {
            const uint2 q = __ldg(reinterpret_cast<const uint2*>(base));
            r.v[0] = q.x; r.v[1] = q.y;
            r.look = __ldg(reinterpret_cast<const uint32_t*>(base + 8));
        }
        r.glo = __ldg(a.gaps + gword);
        r.ghi = __ldg(a.gaps + gword + 1);
    } else {
#pragma unroll
        for (int k = 0; k < 2 * WPL; k++) r.v[k] = 0;
        r.look = r.glo = r.ghi = 0;
    }
    return r;
}

// Called by all 32 lanes of the warp together.
template <int WPL>
__device__ __forceinline__ LaneWindow<WPL> finish_lane(const DecodeArgs& a, const RawLane<WPL>& r, uint32_t tg0,
                                                       uint32_t gshift, uint32_t lane) {
    LaneWindow<WPL> w;
#pragma unroll
    for (int k = 0; k < 2 * WPL; k++) w.w[k] = bswap32(r.v[k]);
    if constexpr (WPL >= 2) {
        const uint32_t next = __shfl_down_sync(0xFFFFFFFFu, r.v[0], 1);  // the next lane's first word
        w.w[2 * WPL] = bswap32(lane == 31 ? r.look : next);
    } else {
        w.w[2 * WPL] = bswap32(r.look);
    }
    w.start = __funnelshift_r(r.glo, r.ghi, gshift) & 31u;
    // every window but the stream's last is whole
    const uint32_t last = a.n_threads - 1;
    const uint32_t whole = tg0 < last ? min(uint32_t(WPL), last - tg0) : 0u;
    const bool has_last = tg0 <= last && last < tg0 + WPL;
    w.wend = 64 * whole + (has_last ? a.last_wend : 0u);
    return w;
}

// Decode the lane's run into its (transposed) slot at shared address slot_s;
// returns the number of codes that start in the run.
template <int WPL, int K>
__device__ __forceinline__ uint32_t decode_lane_once(const LaneWindow<WPL>& w, const Tables& t, uint32_t dtab_s,
                                                     uint32_t slot_s, const uint16_t* ltab, uint32_t long_base,
                                                     uint32_t long_count, bool& bad) {
    // bit position << 16 | 8 x bytes produced; low five bits = placement shift
    uint32_t acc = w.start << 16;
    uint32_t pend = 0, wad = slot_s, idx = 0, ylast = 0;
    for (;;) {
#pragma unroll
        for (int k = 0; k < 2 * WPL; k++)  // one loop per 32 bits, each peeking at one word pair
            decode_half<K, TableLayout<K>::kStride>(acc, pend, wad, idx, ylast, w.w[k], w.w[k + 1],
                                                    min(w.wend, 32u * (k + 1)) << 16, dtab_s);
        if (acc < (kEscape << 16)) break;
        // a code longer than the table: undo the escape, take it from level 2
        acc -= kEscape << 16;
        const uint32_t pos = acc >> 16;
        // the word pair holding bit pos, by selects (an indexed pick would
        // put the window in local memory)
        const uint32_t kw = pos >> 5;
        uint32_t hi = w.w[0], lo = w.w[1];
#pragma unroll
        for (int k = 1; k < 2 * WPL; k++)
            if (kw == uint32_t(k)) {
                hi = w.w[k];
                lo = w.w[k + 1];
            }
        const uint32_t pk = __funnelshift_l(lo, hi, pos);
        const uint32_t li = (pk >> (32 - kLongBits)) - long_base;
        const uint32_t le = li < long_count ? uint32_t(ltab[li]) : 0u;
        int l;
        uint32_t sym;
        if (le) {
            l = int(le >> 8);
            sym = le & 0xFFu;
        } else {
            l = code_length(t.lj_end, pk, K + 1);
            if (!l) {
                bad = true;
                return 0;
            }
            sym = code_symbol(t, pk, l);
        }
        pend |= sym << (acc & 31u);
        const uint32_t before_sym = acc;
        acc += (uint32_t(l) << 16) | 8u;
        if ((acc ^ before_sym) & 32u) {  // the word is complete
            asm volatile("st.shared.u32 [%0], %1;" ::"r"(wad), "r"(pend) : "memory");
            wad += 128;
            pend = 0;
        }
        ylast = 0;
    }
    if (acc & 31u) asm volatile("st.shared.u32 [%0], %1;" ::"r"(wad), "r"(pend) : "memory");
    uint32_t cnt = (acc & 0xFFFFu) >> 3;
    if (ylast) {  // codes of the last table step that start at or past wend
        const uint32_t s = w.wend - ((acc >> 16) - (ylast >> 16));
        if (s < uint32_t(K)) {
            const uint32_t n = (ylast & 0xFFu) >> 3;
            const uint32_t before = __popc(uint32_t(t.mtab[idx]) & ((1u << s) - 1u));
            cnt -= n - min(n, before);
        }
    }
    return cnt;
}

// Copy slot bytes [0, cnt) to staging bytes [pos0, pos0 + cnt): whole words
// from the first word boundary on; returns the slot's first word, whose
// leading bytes go to the positions before that boundary (write_head).  The
// slot is transposed: its words are 32 words apart.
__device__ __forceinline__ uint32_t copy_slot(const uint32_t* slot, uint32_t* stage32, uint32_t pos0, uint32_t cnt) {
    if (cnt == 0) return 0;
    const uint32_t r = (4u - (pos0 & 3u)) & 3u;  // slot byte landing on the first word boundary
    const uint32_t fw = (pos0 + 3) >> 2;
    const uint32_t lw = (pos0 + cnt - 1) >> 2;
    const uint32_t sh = 8 * r;
    const uint32_t first = slot[0];
    uint32_t cur = first;
    uint32_t j = fw;
    const uint32_t* src = slot + 32;
    for (; j + 1 <= lw; j += 2, src += 64) {
        const uint32_t n1 = src[0], n2 = src[32];
        stage32[j] = __funnelshift_r(cur, n1, sh);
        stage32[j + 1] = __funnelshift_r(n1, n2, sh);
        cur = n2;
    }
    if (j <= lw) stage32[j] = __funnelshift_r(cur, src[0], sh);
    return first;
}

// Rounds R .. N-1 of a block's whole-unit merge: round r merges unit
// lane + 32 r from staging bytes 256 r on and stores to dst + 32 r, with the
// offsets as immediates.
template <int R, int N>
__device__ __forceinline__ void merge_rounds(uint32_t ev_s, const uint2 (&sv)[N], uint4* dst, uint32_t m,
                                             uint32_t lane, uint32_t qe) {
    if constexpr (R < N) {
        if (lane + 32 * R < qe) merge_store8<256 * R, 512 * R>(ev_s, sv[R], dst, m);
        merge_rounds<R + 1, N>(ev_s, sv, dst, m, lane, qe);
    }
}

template <int WARPS, int MIN_LEN, int WPL, bool U8, int K>
__global__ void __launch_bounds__(WARPS * 32, 1) decode_warp_kernel(const DecodeArgs a) {
    using L = WarpLayout<MIN_LEN, WPL>;
    using TL = TableLayout<K>;
    // elements per merge unit, 16 output bytes either way
    constexpr uint32_t kUnit = U8 ? 16u : 8u;
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = threadIdx.x >> 5;
    // the gap field of the lane's first window, WPL (32b + lane), lies in the
    // block's 5 WPL gap words
    const uint32_t lane_gword = (5 * WPL * lane) >> 5;
    const uint32_t lane_gshift = (5 * WPL * lane) & 31u;

    // this warp's run of thread blocks [b, b_end); warps are numbered across
    // the CTAs first, so the runs one block longer than the rest (the first
    // n_blocks mod nw) fall at most one per SM instead of filling a few SMs
    // (a stream of few thread blocks runs with fewer warps per CTA, so that
    // its warps spread over all SMs)
    const uint32_t nw = gridDim.x * (blockDim.x >> 5);
    const uint32_t g = warp * gridDim.x + blockIdx.x;
    const uint32_t per = a.n_blocks / nw, extra = a.n_blocks % nw;
    uint32_t b = a.block0 + g * per + (g < extra ? g : extra);
    const uint32_t b_end = b + per + (g < extra ? 1u : 0u);

    __shared__ __align__(8) unsigned long long s_bar;
    __shared__ uint32_t s_abort;
    const uint32_t bar = uint32_t(__cvta_generic_to_shared(&s_bar));
    // the next grid on the stream may start its CTAs as this grid's exit
    // (it waits for this grid before touching memory)
    allow_next_grid();
    // Early staging (the caller's statement that the prior grid writes none
    // of this stream's arrays): the tables and the first block's loads are
    // staged while the prior grid finishes; every write comes after the wait.
    if (!a.early) wait_for_prior_grids();
    if (threadIdx.x == 0) bulk_warp_tables<K>(smem, reinterpret_cast<const uint8_t*>(a.lut), bar);
    copy_narrow_decode<K>(smem, a.lut, int(blockDim.x));
    // the first block's loads overlap the table copy
    RawLane<WPL> nraw{};
    uint32_t noff0 = 0, noff1 = 0;
    if (b < b_end) {
        nraw = load_lane<WPL>(a, WPL * (32 * b + lane), 5 * WPL * b + lane_gword, lane);
        noff0 = __ldg(a.off + b);
        noff1 = __ldg(a.off + b + 1);
    }
    if (threadIdx.x == 0) s_abort = bulk_end(bar) ? 0u : 1u;
    __syncthreads();
    if (a.early) wait_for_prior_grids();
    if (s_abort) {
        if (threadIdx.x == 0 && a.status) atomicOr(a.status, uint32_t(DF11_ERR_CORRUPT));
        return;
    }
    if (!tables_valid(smem, a.status)) return;
    Tables t;
    t.ctab = nullptr;
    t.mtab = reinterpret_cast<const uint16_t*>(smem + TL::kMask);
    t.dtab = reinterpret_cast<const uint2*>(smem + TL::kDecode);
    t.lj_end = reinterpret_cast<const unsigned long long*>(smem + kLutOffLjEnd);
    t.delta = reinterpret_cast<const uint32_t*>(smem + kLutOffDelta);
    t.syms = smem + kLutOffSyms;
    // a replicated table is read through the lane's own copy
    const uint32_t dtab_s = uint32_t(__cvta_generic_to_shared(t.dtab)) + (TL::kNarrow ? 8 * (lane & 15) : 0);
    const uint16_t* ltab = reinterpret_cast<const uint16_t*>(smem + TL::kLong);
    uint32_t long_base, long_count;
    long_table_of<K>(smem, long_base, long_count);
    uint8_t* wbase = smem + TL::kBytes + warp * L::kBytes;
    uint32_t* slot = reinterpret_cast<uint32_t*>(wbase) + lane;
    const uint32_t slot_s = uint32_t(__cvta_generic_to_shared(slot));
    uint8_t* stage = wbase + L::kSlots;
    const uint2* sm8 = reinterpret_cast<const uint2*>(a.sm);
    uint4 carry = make_uint4(0, 0, 0, 0);  // staging bytes of the unit left by the previous block
    bool have_carry = false;
    while (b < b_end) {
        const RawLane<WPL> raw = nraw;
        const uint32_t off0 = noff0, off1 = noff1;
        const bool more = b + 1 < b_end;
        if (more) {  // prefetch the next block (its first position is off1)
            nraw = load_lane<WPL>(a, WPL * (32 * (b + 1) + lane), 5 * WPL * (b + 1) + lane_gword, lane);
            noff0 = off1;
            noff1 = __ldg(a.off + b + 2);
        }
        const bool offs_ok = off0 <= off1 && off1 <= a.n_elems;
        const uint32_t head = off0 & (kUnit - 1);
        // units to store: the head unit (completed by the carried bytes
        // unless this block starts the run), up to the tail unit, which is
        // left to the next block when that block exists and shares it
        const uint32_t u0 = off0 / kUnit;
        const uint32_t u1 = offs_ok ? (off1 + kUnit - 1) / kUnit : u0;
        const bool keep_tail = more && (off1 & (kUnit - 1)) != 0;
        const uint32_t uw = keep_tail && u1 > u0 ? u1 - 1 : u1;
        const bool use_carry = have_carry && head != 0;
        const uint32_t lo = use_carry ? (off0 & ~(kUnit - 1)) : off0;
        // lane q of a merge round r takes unit ub + q + 32 r, with ub = u0
        // rounded down to 16 units (8 for 8-bit symbols), so that every warp
        // access covers whole 128-byte lines (256 sign+mantissa bytes, 512
        // output bytes); lanes whose unit lies before u0 idle in the first round
        const uint32_t a_sh = u0 & (U8 ? 7u : 15u);
        const uint32_t ub = u0 - a_sh;
        // sign+mantissa units requested before the decode: 4 rounds of 32
        // (a 32-window block of LLM weights has ~100 units), 7 for two
        // windows per lane, 13 for four
        constexpr int kPre = WPL == 1 ? 4 : WPL == 2 ? 7 : 13;
        uint2 sv[kPre];
        if constexpr (!U8) {
#pragma unroll
            for (int r = 0; r < kPre; r++)
                sv[r] = ub + lane + 32 * r < uw ? __ldcs(sm8 + ub + lane + 32 * r) : make_uint2(0, 0);
        }

        const LaneWindow<WPL> w = finish_lane<WPL>(a, raw, WPL * (32 * b + lane), lane_gshift, lane);
        bool bad = false;
        const uint32_t cnt = decode_lane_once<WPL, K>(w, t, dtab_s, slot_s, ltab, long_base, long_count, bad);
        uint32_t incl = cnt;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= uint32_t(d)) incl += y;
        }
        // the block's codes must fill exactly its range of output positions
        const bool ok = !bad && offs_ok && (lane != 31 || incl == off1 - off0);
        if (!__all_sync(0xFFFFFFFFu, ok)) {
            if (lane == 0 && a.status) atomicOr(a.status, uint32_t(DF11_ERR_CORRUPT));
            have_carry = false;
        } else {
            if (lane == 0 && use_carry) {
                if constexpr (U8) *reinterpret_cast<uint4*>(stage) = carry;
                else *reinterpret_cast<uint2*>(stage) = make_uint2(carry.x, carry.y);
            }
            __syncwarp();
            const uint32_t pos0 = head + (incl - cnt);
            const uint32_t hword = copy_slot(slot, reinterpret_cast<uint32_t*>(stage), pos0, cnt);
            __syncwarp();
            {  // bytes before this thread's first word boundary
                const uint32_t room = (4u - (pos0 & 3u)) & 3u;
                const uint32_t k = cnt < room ? cnt : room;
                uint8_t* d = stage + pos0;
                if (k > 0) d[0] = uint8_t(hword);
                if (k > 1) d[1] = uint8_t(hword >> 8);
                if (k > 2) d[2] = uint8_t(hword >> 16);
            }
            __syncwarp();
            if constexpr (!U8) {
                const uint2* ev = reinterpret_cast<const uint2*>(stage);
                const uint32_t stage_s = uint32_t(__cvta_generic_to_shared(stage));
                const uint32_t nu = uw - u0;  // units this block stores
                const uint32_t qe = nu + a_sh;  // lanes [a_sh, qe) of the rounds hold them
                const uint32_t m = 0x80808080u;
                if (lo == 8 * u0 && (keep_tail || (off1 & 7u) == 0)) {
                    // every unit is whole (all but the first and last block of a run)
                    const uint32_t ev_s = stage_s + 8 * lane - 8 * a_sh;
                    uint4* dst = reinterpret_cast<uint4*>(a.out) + ub + lane;
                    if (lane >= a_sh && lane < qe) merge_store8<0, 0>(ev_s, sv[0], dst, m);
                    merge_rounds<1, kPre>(ev_s, sv, dst, m, lane, qe);
                    for (uint32_t k = 32 * kPre; lane + k < qe; k += 32)
                        merge_store8(ev_s + 8 * k, __ldcs(sm8 + ub + lane + k), dst + k, m);
                } else {
                    const uint32_t uf = (lo + 7) >> 3, ul = off1 >> 3;  // whole units: [uf, ul)
                    auto unit = [&](uint32_t q, const uint2 s8) {  // unit u0 + q - a_sh
                        const uint32_t k = q - a_sh, u = u0 + k;
                        if (u >= uf && u < ul)
                            merge_store8(stage_s + 8 * k, s8, reinterpret_cast<uint4*>(a.out) + u, m);
                        else
                            merge_unit(ev[k], s8, u, lo, off1, a.out);
                    };
    #pragma unroll
                    for (int r = 0; r < kPre; r++)
                        if (lane + 32 * r >= a_sh && lane + 32 * r < qe) unit(lane + 32 * r, sv[r]);
                    for (uint32_t q = lane + 32 * kPre; q < qe; q += 32) unit(q, __ldcs(sm8 + ub + q));
                }
                if (keep_tail) {
                    const uint2 c = ev[u1 - 1 - u0];
                    carry = make_uint4(c.x, c.y, 0, 0);
                }
            } else {
                // 8-bit symbols: the staged bytes themselves, rotated back
                const uint4* ev16 = reinterpret_cast<const uint4*>(stage);
                const uint32_t nu = uw - u0;  // units this block stores
                const uint32_t qe = nu + a_sh;
                uint4* out16 = reinterpret_cast<uint4*>(a.out8);
                if (lo == kUnit * u0 && (keep_tail || (off1 & (kUnit - 1)) == 0)) {
                    for (uint32_t q = lane; q < qe; q += 32)
                        if (q >= a_sh) __stcs(out16 + ub + q, unrotate16(ev16[q - a_sh]));
                } else {
                    for (uint32_t q = lane; q < qe; q += 32) {
                        if (q < a_sh) continue;
                        const uint32_t k = q - a_sh, u = u0 + k;
                        const uint4 v = unrotate16(ev16[k]);
                        const uint32_t i0 = kUnit * u;
                        if (i0 >= lo && i0 + kUnit <= off1) {
                            __stcs(out16 + u, v);
                        } else {
                            const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int e = 0; e < 16; e++)
                                if (i0 + e >= lo && i0 + e < off1) a.out8[i0 + e] = uint8_t(words[e >> 2] >> (8 * (e & 3)));
                        }
                    }
                }
                if (keep_tail) carry = ev16[u1 - 1 - u0];
            }
            have_carry = keep_tail;
        }
        __syncwarp();
        b++;
    }
}

// ---------------------------------------------------------------------------
// Independent chunks, an ablation of the gap-and-scan design (the parallel
// decoding of "EntroLLM: Compressao de Pesos Codificada por Entropia ...",
// section "Metodologia", item 3, segments the coded weights so that segments
// decode independently): the stream records the start bit of every
// kIndChunk-element chunk instead of Gaps and block offsets, so a lane
// decodes its chunk with no gap, count or prefix sum and writes exactly
// kIndChunk symbols to a fixed slot.  A warp takes 32 consecutive chunks and
// first stages their stream words in shared memory.
// ---------------------------------------------------------------------------
struct ChunkArgs {
    const uint32_t* exp32;      // EncodedExponent as 32-bit words (stream byte order)
    const uint2* sm8;           // PackedSignMantissa, 8 bytes per unit
    const uint32_t* chunk_bit;  // start bit of each chunk, then total_bits
    const uint4* lut;
    uint16_t* out;
    uint32_t* status;
    uint32_t n_elems;
    uint32_t n_chunks;
    uint32_t exp_words;  // words of EncodedExponent that may be read
};

constexpr int kChunkWarps = 12;
// 32 chunks of codes of at most 32 bits, plus the peek's lookahead word
constexpr uint32_t kChunkStreamWords = 32 * kIndChunk + 4;
// staged symbols per lane: the chunk plus up to 3 decoded past it, 8-byte aligned
constexpr uint32_t kChunkSlot = kIndChunk + 8;
constexpr uint32_t kChunkWarpBytes = 4 * kChunkStreamWords + 32 * kChunkSlot;
static_assert(kChunkWarpBytes % 16 == 0 && kChunkSlot % 8 == 0, "aligned per-warp buffers");

__global__ void __launch_bounds__(kChunkWarps * 32, 1) decode_chunk_kernel(const ChunkArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ __align__(8) unsigned long long s_bar;
    __shared__ uint32_t s_abort;
    const uint32_t bar = uint32_t(__cvta_generic_to_shared(&s_bar));
    wait_for_prior_grids();
    if (threadIdx.x == 0) {
        bulk_warp_tables<kPeekBits>(smem, reinterpret_cast<const uint8_t*>(a.lut), bar);
        s_abort = bulk_end(bar) ? 0u : 1u;
    }
    __syncthreads();
    if (s_abort) {
        if (threadIdx.x == 0 && a.status) atomicOr(a.status, uint32_t(DF11_ERR_CORRUPT));
        return;
    }
    if (!tables_valid(smem, a.status)) return;
    Tables t;
    t.ctab = nullptr;
    t.mtab = reinterpret_cast<const uint16_t*>(smem + kCompactMask);
    t.dtab = reinterpret_cast<const uint2*>(smem + kCompactDecode);
    t.lj_end = reinterpret_cast<const unsigned long long*>(smem + kLutOffLjEnd);
    t.delta = reinterpret_cast<const uint32_t*>(smem + kLutOffDelta);
    t.syms = smem + kLutOffSyms;
    const uint16_t* ltab = reinterpret_cast<const uint16_t*>(smem + kCompactLong);
    const uint32_t long_base = reinterpret_cast<const LutHeader*>(smem)->long_base;
    const uint32_t long_count = reinterpret_cast<const LutHeader*>(smem)->long_count;
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = threadIdx.x >> 5;
    uint32_t* s_stream = reinterpret_cast<uint32_t*>(smem + kCompactBytes + warp * kChunkWarpBytes);
    uint8_t* s_slot = reinterpret_cast<uint8_t*>(s_stream + kChunkStreamWords);
    uint32_t* my_slot = reinterpret_cast<uint32_t*>(s_slot + lane * kChunkSlot);
    const uint32_t slot_s = uint32_t(__cvta_generic_to_shared(s_slot));
    const uint32_t n_groups = (a.n_chunks + 31) / 32;
    const uint32_t stride = gridDim.x * kChunkWarps;
    // one group's start bits, and the first kPreWords of its stream words
    constexpr uint32_t kPreWords = 8;  // per lane: 256 words cover a typical group
    struct GroupBits {
        uint32_t b0, b1, my0, my1;
    };
    auto load_bits = [&](uint32_t g) {
        GroupBits r{0, 0, 0, 0};
        if (g < n_groups) {
            const uint32_t k = 32 * g + lane, kl = min(32 * g + 32, a.n_chunks);
            r.b0 = __ldg(a.chunk_bit + 32 * g);
            r.b1 = __ldg(a.chunk_bit + kl);
            r.my0 = k < a.n_chunks ? __ldg(a.chunk_bit + k) : r.b1;
            r.my1 = k < a.n_chunks ? __ldg(a.chunk_bit + k + 1) : r.b1;
        }
        return r;
    };
    auto word_range = [&](const GroupBits& gb, uint32_t& w0, uint32_t& w_end) {
        w0 = gb.b0 >> 5;
        w_end = min((gb.b1 >> 5) + 2, a.exp_words);
    };
    auto load_words = [&](const GroupBits& gb, uint32_t (&wv)[kPreWords]) {
        uint32_t w0, w_end;
        word_range(gb, w0, w_end);
#pragma unroll
        for (int r = 0; r < int(kPreWords); r++) {
            const uint32_t j = lane + 32 * r;
            wv[r] = w_end > w0 && j < w_end - w0 ? __ldg(a.exp32 + w0 + j) : 0u;
        }
    };
    uint32_t g = warp * gridDim.x + blockIdx.x;
    GroupBits nbits = load_bits(g);
    uint32_t nwv[kPreWords];
    load_words(nbits, nwv);
    for (; g < n_groups; g += stride) {
        const GroupBits gb = nbits;
        uint32_t wv[kPreWords];
#pragma unroll
        for (int r = 0; r < int(kPreWords); r++) wv[r] = nwv[r];
        nbits = load_bits(g + stride);  // in flight during this group's work
        const uint32_t k = 32 * g + lane;
        const uint32_t b0 = gb.b0, b1 = gb.b1, my0 = gb.my0, my1 = gb.my1;
        uint32_t w0, w_end;
        word_range(gb, w0, w_end);
        // (every index into the staged words below stays inside them)
        bool bad = b1 < b0 || my0 < b0 || my1 < my0 || my1 > b1 || w_end <= w0 || w_end - w0 > kChunkStreamWords ||
                   (my0 >> 5) >= w_end;
        if (__any_sync(0xFFFFFFFFu, bad)) {
            if (lane == 0 && a.status) atomicOr(a.status, uint32_t(DF11_ERR_CORRUPT));
            load_words(nbits, nwv);
            continue;
        }
        const uint32_t nwords = w_end - w0;
#pragma unroll
        for (int r = 0; r < int(kPreWords); r++) {
            const uint32_t j = lane + 32 * r;
            if (j < nwords) s_stream[j] = bswap32(wv[r]);
        }
        for (uint32_t j = lane + 32 * kPreWords; j < nwords; j += 32) s_stream[j] = bswap32(__ldg(a.exp32 + w0 + j));
        // this group's sign+mantissa units (32 kIndChunk / 8 over 32 lanes),
        // requested before the decode
        const uint32_t e0 = 32 * g * kIndChunk;
        const uint32_t e1 = min(a.n_elems, e0 + 32 * kIndChunk);
        const uint32_t nunits = (e1 - e0 + 7) / 8;
        uint2 sv[kIndChunk / 8];
#pragma unroll
        for (int r = 0; r < int(kIndChunk / 8); r++) {
            const uint32_t q = lane + 32 * r;
            sv[r] = q < nunits ? __ldcs(a.sm8 + e0 / 8 + q) : make_uint2(0, 0);
        }
        __syncwarp();
        // this lane's chunk: exactly cnt codes from bit my0
        const uint32_t cnt = k < a.n_chunks ? min(kIndChunk, a.n_elems - k * kIndChunk) : 0u;
        const uint32_t rel = my0 - 32 * w0;
        uint32_t wi = rel >> 5, pos = rel & 31u;
        uint32_t hi = s_stream[wi], lo = wi + 1 < nwords ? s_stream[wi + 1] : 0u;
        uint32_t produced = 0, pend = 0;
        for (uint32_t steps = 0; produced < cnt; steps++) {
            if (steps >= kIndChunk) {  // every step decodes at least one code
                bad = true;
                break;
            }
            const uint32_t pk = __funnelshift_l(lo, hi, pos);
            const uint2 e = t.dtab[pk >> (32 - kPeekBits)];
            uint32_t x, nsym, used;
            if ((e.y >> 16) >= kEscape) {  // a code longer than the table
                const uint32_t li = (pk >> (32 - kLongBits)) - long_base;
                const uint32_t le = li < long_count ? uint32_t(ltab[li]) : 0u;
                if (le) {
                    used = le >> 8;
                    x = le & 0xFFu;
                } else {
                    used = uint32_t(code_length(t.lj_end, pk, kPeekBits + 1));
                    if (!used) {
                        bad = true;
                        break;
                    }
                    x = code_symbol(t, pk, int(used));
                }
                nsym = 1;
            } else {
                x = e.x;
                nsym = (e.y & 0xFFu) >> 3;
                used = e.y >> 16;
            }
            // append nsym symbol bytes at byte `produced` of the slot
            const uint32_t sh = 8 * (produced & 3u);
            pend |= x << sh;
            if ((produced & 3u) + nsym >= 4) {
                my_slot[produced >> 2] = pend;
                pend = sh ? x >> (32 - sh) : 0u;
            }
            produced += nsym;
            pos += used;
            while (pos >= 32) {
                hi = lo;
                wi++;
                lo = wi + 1 < nwords ? s_stream[wi + 1] : 0u;
                pos -= 32;
            }
            if (wi >= nwords) {
                bad = true;
                break;
            }
        }
        if (produced & 3u) my_slot[produced >> 2] = pend;
        // a chunk decoded without symbols past its end stops at the next start
        if (produced == cnt && cnt && 32 * (w0 + wi) + pos != my1) bad = true;
        load_words(nbits, nwv);  // the next group's words, in flight during the merge
        if (__any_sync(0xFFFFFFFFu, bad)) {
            if (lane == 0 && a.status) atomicOr(a.status, uint32_t(DF11_ERR_CORRUPT));
            __syncwarp();
            continue;
        }
        __syncwarp();
        // merge the group's elements [e0, e1) in 8-element units
#pragma unroll
        for (int r = 0; r < int(kIndChunk / 8); r++) {
            const uint32_t q = lane + 32 * r;
            if (q >= nunits) break;
            const uint32_t off = (q / (kIndChunk / 8)) * kChunkSlot + 8 * (q % (kIndChunk / 8));
            const uint32_t u = e0 / 8 + q;
            if (e0 + 8 * q + 8 <= e1)
                merge_store8(slot_s + off, sv[r], reinterpret_cast<uint4*>(a.out) + u, 0x80808080u);
            else
                merge_unit(*reinterpret_cast<const uint2*>(s_slot + off), sv[r], u, e0, e1, a.out);
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// T >= 64: one CTA of T threads decodes one thread block per iteration, with
// a block-wide scan.
// ---------------------------------------------------------------------------
template <int T>
constexpr size_t block_stage_bytes() {
    return 64 * T + 64;
}

template <int T>
__global__ void __launch_bounds__(T) decode_block_kernel(const DecodeArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ __align__(8) unsigned long long s_bar;
    __shared__ uint32_t s_abort;
    const uint32_t bar = uint32_t(__cvta_generic_to_shared(&s_bar));
    wait_for_prior_grids();
    if (threadIdx.x == 0) {
        bulk_begin(bar, uint32_t(kLutWideBytes));
        bulk_copy(uint32_t(__cvta_generic_to_shared(smem)), a.lut, uint32_t(kLutWideBytes), bar);
        s_abort = bulk_end(bar) ? 0u : 1u;
    }
    uint8_t* stage = smem + kLutWideBytes;
    uint32_t* s_warp = reinterpret_cast<uint32_t*>(stage + block_stage_bytes<T>());
    __syncthreads();
    if (s_abort) {
        if (threadIdx.x == 0 && a.status) atomicOr(a.status, uint32_t(DF11_ERR_CORRUPT));
        return;
    }
    if (!tables_valid(smem, a.status)) return;
    const Tables t = tables_at(smem);
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = threadIdx.x >> 5;
    const uint32_t my_gword = (5 * threadIdx.x) >> 5;
    const uint32_t my_gshift = (5 * threadIdx.x) & 31u;
    constexpr uint32_t kGwordsPerBlock = 5 * T / 32;

    const uint32_t b_end = a.block0 + a.n_blocks;
    uint32_t b = a.block0 + blockIdx.x;
    RawWindow nraw{};
    uint32_t noff0 = 0, noff1 = 0;
    if (b < b_end) {
        nraw = load_window(a, T * b + threadIdx.x, kGwordsPerBlock * b + my_gword);
        noff0 = __ldg(a.off + b);
        noff1 = __ldg(a.off + b + 1);
    }
    while (b < b_end) {
        const RawWindow raw = nraw;
        const uint32_t off0 = noff0, off1 = noff1;
        const uint32_t bn = b + gridDim.x;
        if (bn < b_end) {
            nraw = load_window(a, T * bn + threadIdx.x, kGwordsPerBlock * bn + my_gword);
            noff0 = __ldg(a.off + bn);
            noff1 = __ldg(a.off + bn + 1);
        }
        const bool offs_ok = off0 <= off1 && off1 <= a.n_elems;
        const uint32_t c0 = off0 >> 4;
        const uint32_t c1 = offs_ok ? (off1 + 15) >> 4 : c0;
        uint4 s0 = make_uint4(0, 0, 0, 0);
        if (c0 + threadIdx.x < c1) s0 = __ldcs(a.sm + c0 + threadIdx.x);

        const Window w = finish_window(a, raw, T * b + threadIdx.x, my_gshift);
        bool bad = false;
        const uint32_t cnt = count_codes(w, t, bad);
        uint32_t incl = cnt;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= uint32_t(d)) incl += y;
        }
        if (lane == 31) s_warp[warp] = incl;
        const int any_bad = __syncthreads_or(bad);
        uint32_t before = 0, total = 0;
#pragma unroll
        for (int k = 0; k < T / 32; k++) {
            const uint32_t v = s_warp[k];
            total += v;
            before += (uint32_t(k) < warp) ? v : 0u;
        }
        if (any_bad || !block_consistent(off0, off1, total, a.n_elems)) {
            if (threadIdx.x == 0 && a.status) atomicOr(a.status, uint32_t(DF11_ERR_CORRUPT));
        } else {
            const uint32_t pos0 = (off0 & 15u) + before + incl - cnt;
            const uint32_t hword = decode_codes(w, t, reinterpret_cast<uint32_t*>(stage), pos0, cnt);
            __syncthreads();
            write_head(stage, pos0, cnt, hword);
            __syncthreads();
            const uint4* ev = reinterpret_cast<const uint4*>(stage);
            if (c0 + threadIdx.x < c1) merge_chunk(ev[threadIdx.x], s0, c0 + threadIdx.x, off0, off1, a.out);
            for (uint32_t k = threadIdx.x + T; c0 + k < c1; k += T)
                merge_chunk(ev[k], __ldcs(a.sm + c0 + k), c0 + k, off0, off1, a.out);
        }
        __syncthreads();
        b = bn;
    }
}

struct LaunchInfo {
    std::atomic<int> ready{0};
    int per_sm = 0;
    int sms = 0;
};
constexpr int kMaxDev = 64;
LaunchInfo g_info[kMaxDev][32];  // [device][variant]: BF16 0..15, 8-bit symbols 16..31

// One CTA per SM: all warps share one copy of the tables.  With one window
// per lane, 32 warps at 64 registers measured faster than two CTAs of 20
// warps at 48 registers.
constexpr int kWarpsLong = 32;   // some code is 1 bit long
constexpr int kWarpsShort = 32;  // every code has 2 bits or more
// two windows per lane: 28 warps leave 72 registers per thread (the merge's
// seven prefetched rounds fit) and measured faster than 24, 26, 30 or 32
constexpr int kWarpsTwoWindows = 28;
// 8-bit symbols (60 registers, no sign+mantissa prefetch) with codes of 4
// bits or more: slots and staging for 32 codes per lane, so 32 warps fit
// (2.8% faster than 28 on the quantized Llama-3.1-8B block)
constexpr int kWarpsTwoWindowsU8 = 32;
// four windows per lane with 2-bit codes: 8,384 bytes of slots and staging
// per warp, so 20 warps fit beside the tables
constexpr int kWarpsFourWindows = 20;
// two windows per lane with a 1-bit code: the same 8,384 bytes per warp
constexpr int kWarpsTwoWindowsOneBit = 20;

// How one stream is decoded: which kernel, its CTA shape and its shared
// memory.  Warp kernels take up to `warps` warps per CTA, one CTA per SM; a
// stream with fewer thread blocks than warps x SMs gets ceil(blocks / SMs)
// warps per CTA so that it still spreads over every SM.  Block kernels take T
// threads per CTA.
struct Plan {
    const void* kernel;
    int slot;            // LaunchInfo slot
    uint32_t warps;      // warp kernels: warps per CTA at most; 0 for block kernels
    uint32_t threads;    // block kernels: T
    size_t smem_fixed;   // tables (+ block kernels' staging)
    size_t smem_per_warp;
    uint32_t peek_bits, copies;
    char name[64];
};

template <int WARPS, int MIN_LEN, int WPL, bool U8, int K = kPeekBits>
Plan warp_plan(int slot) {
    using TL = TableLayout<K>;
    static_assert(TL::kBytes + size_t(WARPS) * WarpLayout<MIN_LEN, WPL>::kBytes <= 227 * 1024,
                  "shared memory per CTA");
    Plan p{};
    p.kernel = reinterpret_cast<const void*>(&decode_warp_kernel<WARPS, MIN_LEN, WPL, U8, K>);
    p.slot = slot + (U8 ? 16 : 0);
    p.warps = WARPS;
    p.smem_fixed = TL::kBytes;
    p.smem_per_warp = WarpLayout<MIN_LEN, WPL>::kBytes;
    p.peek_bits = K;
    p.copies = TL::kRep;
    std::snprintf(p.name, sizeof(p.name), "decode_warp_kernel<%d,%d,%d,%d,%d>", WARPS, MIN_LEN, WPL, int(U8), K);
    return p;
}

template <int T>
Plan block_plan(int slot) {
    Plan p{};
    p.kernel = reinterpret_cast<const void*>(&decode_block_kernel<T>);
    p.slot = slot;
    p.threads = T;
    p.smem_fixed = kLutWideBytes + block_stage_bytes<T>() + 4 * (T / 32);
    p.peek_bits = kPeekBits;
    p.copies = 1;
    std::snprintf(p.name, sizeof(p.name), "decode_block_kernel<%d>", T);
    return p;
}

struct Shape {
    unsigned grid, block;
    size_t smem;
};

// Grid and CTA shape of a plan for n_blocks thread blocks on at most max_sms
// SMs of the current device (first use per device and kernel: sets the
// kernel's shared-memory limit and queries its occupancy).
df11_status shape_of(const Plan& p, uint64_t n_blocks, const df11_decode_options& o, Shape* out) {
    const uint32_t max_sms = o.max_sms ? o.max_sms : UINT32_MAX;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return fail(DF11_ERR_CUDA, "cudaGetDevice failed");
    const size_t smem_max = p.smem_fixed + (p.warps ? p.warps * p.smem_per_warp : 0);
    const int threads_max = p.warps ? int(32 * p.warps) : int(p.threads);
    LaunchInfo& li = g_info[dev][p.slot];
    if (!li.ready.load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(p.kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_max));
        if (e != cudaSuccess) return fail(DF11_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        int per_sm = 0, sms = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, p.kernel, threads_max, smem_max);
        if (e != cudaSuccess) return fail(DF11_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(e));
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return fail(DF11_ERR_CUDA, "SM count: %s", cudaGetErrorString(e));
        li.per_sm = per_sm > 0 ? per_sm : 1;
        li.sms = sms;
        li.ready.store(1, std::memory_order_release);
    }
    const uint64_t sms = max_sms < uint32_t(li.sms) ? max_sms : uint32_t(li.sms);
    if (!p.warps) {
        const uint64_t want = o.ctas ? uint64_t(o.ctas) : uint64_t(li.per_sm) * sms;
        *out = Shape{unsigned(n_blocks < want ? n_blocks : want), p.threads, p.smem_fixed};
        return DF11_OK;
    }
    // The slowest warp decodes ceil(n_blocks / all warps) thread blocks; the
    // fewest warps per CTA that keep that count let each of them run faster
    // (a stream of 38 K blocks: 26 warps per SM doing 10 blocks each instead
    // of 28 doing 9 or 10).  Few blocks: fewer warps per CTA, every SM.
    const uint64_t cap = o.max_warps_per_cta && o.max_warps_per_cta < p.warps ? o.max_warps_per_cta : p.warps;
    uint64_t warps = cap;
    const uint64_t per = (n_blocks + warps * sms - 1) / (warps * sms);
    if (per > 0) warps = ((n_blocks + per - 1) / per + sms - 1) / sms;
    if (warps > cap) warps = cap;
    if (warps < 1) warps = 1;
    const uint64_t ctas = (n_blocks + warps - 1) / warps;
    const uint64_t want = o.ctas ? uint64_t(o.ctas) : uint64_t(li.per_sm) * sms;
    *out = Shape{unsigned(ctas < want ? ctas : want), unsigned(32 * warps), p.smem_fixed + warps * p.smem_per_warp};
    return DF11_OK;
}

// Forget a kernel's set-up on the current device: the next launch sets its
// shared-memory limit again.  A device reset, or another context on the same
// device, loads the module again with the attribute back at its default.
void forget_setup(const Plan& p) {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDev)
        g_info[dev][p.slot].ready.store(0, std::memory_order_release);
}

df11_status launch_plan(const Plan& p, const DecodeArgs& a, const df11_decode_options& o, cudaStream_t stream,
                        bool retried = false) {
    Shape sh;
    df11_status st = shape_of(p, a.n_blocks, o, &sh);
    if (st != DF11_OK) return st;
    DecodeArgs args = a;
    void* params[] = {&args};
    // programmatic stream serialisation: the CTAs may be placed while the
    // previous kernel on the stream drains; each waits for it (and its
    // memory) before reading anything
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sh.grid);
    cfg.blockDim = dim3(sh.block);
    cfg.dynamicSmemBytes = sh.smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelExC(&cfg, p.kernel, params);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess && !retried) {  // a stale set-up: redo it once
        forget_setup(p);
        return launch_plan(p, a, o, stream, true);
    }
    if (e != cudaSuccess) return fail(DF11_ERR_CUDA, "decode launch (%s): %s", p.name, cudaGetErrorString(e));
    return DF11_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

// Checks a header against the format's own arithmetic (used by decompress
// and encode before any launch).
df11_status check_header(const df11_header* h) {
    if (!h) return fail(DF11_ERR_INVALID, "null header");
    if (h->version != DF11_VERSION) return fail(DF11_ERR_INVALID, "header version %u", h->version);
    if (h->window_bytes != DF11_WINDOW_BYTES) return fail(DF11_ERR_INVALID, "window_bytes %u", h->window_bytes);
    const uint32_t T = h->threads_per_block;
    if (T < 32 || T > 1024 || (T & (T - 1))) return fail(DF11_ERR_INVALID, "threads_per_block %u", T);
    if (h->n_elems >= (uint64_t(1) << 32)) return fail(DF11_ERR_TOO_LARGE, "n_elems >= 2^32");
    df11_header ref = *h;
    fill_sizes(&ref);
    if (ref.n_threads != h->n_threads || ref.n_blocks != h->n_blocks || ref.bytes_exp != h->bytes_exp ||
        ref.bytes_sm != h->bytes_sm || ref.bytes_gaps != h->bytes_gaps || ref.bytes_off != h->bytes_off ||
        ref.bytes_lut != h->bytes_lut)
        return fail(DF11_ERR_INVALID, "header sizes disagree with n_elems/total_bits/threads_per_block");
    if (h->n_elems && (h->total_bits < h->n_elems || h->total_bits > 32 * h->n_elems))
        return fail(DF11_ERR_INVALID, "total_bits inconsistent with n_elems");
    return DF11_OK;
}

}  // namespace df11

using namespace df11;

namespace df11 {
namespace {

// The decode kernel for a stream.  T = 64 (the library default) and codes of
// at least 2 bits: the warp kernel with two windows per lane.  T = 32: one
// window per lane.  T = 64 with a 1-bit code (a lane could then hold 128
// codes, too many for its slot) and T >= 128: the block kernel, whose two
// decode passes need no slot.
df11_status plan_for(const char* fn, const df11_header* hdr, bool u8, uint32_t peek_bits, Plan* out) {
    if (peek_bits != 0 && peek_bits != uint32_t(kPeekBits) &&
        (u8 || hdr->threads_per_block != 64 || peek_bits < 8 || peek_bits > 10))
        return fail(DF11_ERR_INVALID, "%s: peek_bits %u (8, 9 or 10 only for BF16 streams with T = 64)", fn,
                    peek_bits);
    uint32_t min_len = 32;
    for (int v = 0; v < 256; v++)
        if (hdr->code_len[v] && hdr->code_len[v] < min_len) min_len = hdr->code_len[v];
    const uint32_t T = hdr->threads_per_block;
    if (u8) {  // the warp kernel only
        if (T == 32) {
            *out = min_len >= 2 ? warp_plan<kWarpsShort, 2, 1, true>(6) : warp_plan<kWarpsLong, 1, 1, true>(0);
            return DF11_OK;
        }
        if (T == 64 && min_len >= 4) {
            *out = warp_plan<kWarpsTwoWindowsU8, 4, 2, true>(8);
            return DF11_OK;
        }
        if (T == 64) {
            *out = min_len >= 2 ? warp_plan<kWarpsTwoWindows, 2, 2, true>(7)
                                : warp_plan<kWarpsTwoWindowsOneBit, 1, 2, true>(13);
            return DF11_OK;
        }
        if (T == 128 && min_len >= 2) {  // four windows per lane
            *out = min_len >= 4 ? warp_plan<kWarpsTwoWindows, 4, 4, true>(14)
                                : warp_plan<kWarpsFourWindows, 2, 4, true>(15);
            return DF11_OK;
        }
        return fail(DF11_ERR_INVALID,
                    "%s: streams of 8-bit symbols decode with T = 32 or 64, or 128 when no code is 1 bit long",
                    fn);
    }
    switch (T) {
        case 32:
            *out = min_len >= 2 ? warp_plan<kWarpsShort, 2, 1, false>(6) : warp_plan<kWarpsLong, 1, 1, false>(0);
            return DF11_OK;
        case 64:
            if (min_len >= 2) {
                // the narrow first-level tables, 16 copies each (an ablation:
                // slower on LLM weights, see df11_decode_options)
                if (peek_bits == 10) *out = warp_plan<20, 2, 2, false, 10>(10);
                else if (peek_bits == 9) *out = warp_plan<kWarpsTwoWindows, 2, 2, false, 9>(11);
                else if (peek_bits == 8) *out = warp_plan<kWarpsTwoWindows, 2, 2, false, 8>(12);
                else *out = warp_plan<kWarpsTwoWindows, 2, 2, false>(7);
                return DF11_OK;
            }
            if (peek_bits && peek_bits != uint32_t(kPeekBits))
                return fail(DF11_ERR_INVALID, "%s: narrow tables need codes of 2 bits or more", fn);
            // a 1-bit code: slots and staging for 128 codes per lane
            *out = warp_plan<kWarpsTwoWindowsOneBit, 1, 2, false>(13);
            return DF11_OK;
        case 128:  // four windows per lane when every code has 2 bits or more
            *out = min_len >= 2 ? warp_plan<kWarpsFourWindows, 2, 4, false>(14) : block_plan<128>(2);
            return DF11_OK;
        case 256: *out = block_plan<256>(3); return DF11_OK;
        case 512: *out = block_plan<512>(4); return DF11_OK;
        case 1024: *out = block_plan<1024>(5); return DF11_OK;
        default: return fail(DF11_ERR_INVALID, "threads_per_block %u", T);
    }
}

// BF16 streams (u8 = false): d_sm read, d_out holds n_elems uint16; streams
// of 8-bit symbols (u8 = true): no d_sm, d_out holds n_elems bytes.
df11_status decompress_on(const char* fn, bool u8, const df11_header* hdr, const uint8_t* d_exp,
                          const uint8_t* d_sm, const uint8_t* d_gaps, const uint32_t* d_block_off,
                          const void* d_lut, void* d_out, uint32_t* d_status, const df11_decode_options& opt,
                          void* stream, uint64_t block_begin = 0, uint64_t block_end = UINT64_MAX) {
    df11_status st = check_header(hdr);
    if (st != DF11_OK) return st;
    if (block_end == UINT64_MAX) block_end = hdr->n_blocks;
    if (block_begin > block_end || block_end > hdr->n_blocks)
        return fail(DF11_ERR_INVALID, "%s: block range [%llu, %llu) outside [0, %llu)", fn,
                    (unsigned long long)block_begin, (unsigned long long)block_end,
                    (unsigned long long)hdr->n_blocks);
    if (hdr->n_elems == 0 || block_begin == block_end) return DF11_OK;
    if (!d_exp || (!u8 && !d_sm) || !d_gaps || !d_block_off || !d_lut || !d_out)
        return fail(DF11_ERR_INVALID, "%s: null device pointer", fn);
    if (!aligned16(d_exp) || (!u8 && !aligned16(d_sm)) || !aligned16(d_gaps) || !aligned16(d_block_off) ||
        !aligned16(d_lut) || !aligned16(d_out))
        return fail(DF11_ERR_INVALID, "%s: device pointers must be 16-byte aligned", fn);
    DecodeArgs a;
    a.exp = d_exp;
    a.sm = reinterpret_cast<const uint4*>(d_sm);
    a.gaps = reinterpret_cast<const uint32_t*>(d_gaps);
    a.off = d_block_off;
    a.lut = reinterpret_cast<const uint4*>(d_lut);
    a.out = u8 ? nullptr : static_cast<uint16_t*>(d_out);
    a.out8 = u8 ? static_cast<uint8_t*>(d_out) : nullptr;
    a.status = d_status;
    a.n_elems = uint32_t(hdr->n_elems);
    a.n_threads = uint32_t(hdr->n_threads);
    a.block0 = uint32_t(block_begin);
    a.n_blocks = uint32_t(block_end - block_begin);
    a.last_wend = uint32_t(hdr->total_bits - 64 * (hdr->n_threads - 1));
    a.early = opt.early_staging;
    Plan p;
    st = plan_for(fn, hdr, u8, opt.peek_bits, &p);
    if (st != DF11_OK) return st;
    return launch_plan(p, a, opt, reinterpret_cast<cudaStream_t>(stream));
}

constexpr df11_decode_options kDefaultOptions{0, 0, 0, 0, 0, 0, 0, 0};

}  // namespace
}  // namespace df11

extern "C" df11_status df11_decompress(const df11_header* hdr, const uint8_t* d_exp, const uint8_t* d_sm,
                                       const uint8_t* d_gaps, const uint32_t* d_block_off,
                                       const void* d_lut, uint16_t* d_out, uint32_t* d_status,
                                       void* stream) {
    return decompress_on("df11_decompress", false, hdr, d_exp, d_sm, d_gaps, d_block_off, d_lut, d_out, d_status,
                         kDefaultOptions, stream);
}

extern "C" df11_status df11_decompress_sms(const df11_header* hdr, const uint8_t* d_exp, const uint8_t* d_sm,
                                           const uint8_t* d_gaps, const uint32_t* d_block_off,
                                           const void* d_lut, uint16_t* d_out, uint32_t* d_status,
                                           uint32_t max_sms, void* stream) {
    if (max_sms == 0) return fail(DF11_ERR_INVALID, "df11_decompress_sms: max_sms must be at least 1");
    df11_decode_options o = kDefaultOptions;
    o.max_sms = max_sms;
    return decompress_on("df11_decompress_sms", false, hdr, d_exp, d_sm, d_gaps, d_block_off, d_lut, d_out,
                         d_status, o, stream);
}

extern "C" df11_status df11_decompress_opts(const df11_header* hdr, const uint8_t* d_exp, const uint8_t* d_sm,
                                            const uint8_t* d_gaps, const uint32_t* d_block_off,
                                            const void* d_lut, void* d_out, uint32_t symbols_u8,
                                            const df11_decode_options* opt, uint32_t* d_status, void* stream) {
    if (!opt) return fail(DF11_ERR_INVALID, "df11_decompress_opts: null options");
    if (opt->reserved) return fail(DF11_ERR_INVALID, "df11_decompress_opts: reserved field must be zero");
    if (opt->early_staging > 1) return fail(DF11_ERR_INVALID, "df11_decompress_opts: early_staging is 0 or 1");
    if (opt->block_begin || opt->block_end)
        return decompress_on("df11_decompress_opts", symbols_u8 != 0, hdr, d_exp, d_sm, d_gaps, d_block_off, d_lut,
                             d_out, d_status, *opt, stream, opt->block_begin, opt->block_end);
    return decompress_on("df11_decompress_opts", symbols_u8 != 0, hdr, d_exp, d_sm, d_gaps, d_block_off, d_lut,
                         d_out, d_status, *opt, stream);
}

extern "C" df11_status df11_decompress_u8(const df11_header* hdr, const uint8_t* d_exp, const uint8_t* d_gaps,
                                          const uint32_t* d_block_off, const void* d_lut, uint8_t* d_out,
                                          uint32_t* d_status, void* stream) {
    return decompress_on("df11_decompress_u8", true, hdr, d_exp, nullptr, d_gaps, d_block_off, d_lut, d_out,
                         d_status, kDefaultOptions, stream);
}

extern "C" df11_status df11_decompress_blocks(const df11_header* hdr, const uint8_t* d_exp, const uint8_t* d_sm,
                                              const uint8_t* d_gaps, const uint32_t* d_block_off,
                                              const void* d_lut, uint16_t* d_out, uint64_t block_begin,
                                              uint64_t block_end, uint32_t* d_status, void* stream) {
    return decompress_on("df11_decompress_blocks", false, hdr, d_exp, d_sm, d_gaps, d_block_off, d_lut, d_out,
                         d_status, kDefaultOptions, stream, block_begin, block_end);
}

extern "C" df11_status df11_decompress_u8_blocks(const df11_header* hdr, const uint8_t* d_exp, const uint8_t* d_gaps,
                                                 const uint32_t* d_block_off, const void* d_lut, uint8_t* d_out,
                                                 uint64_t block_begin, uint64_t block_end, uint32_t* d_status,
                                                 void* stream) {
    return decompress_on("df11_decompress_u8_blocks", true, hdr, d_exp, nullptr, d_gaps, d_block_off, d_lut,
                         d_out, d_status, kDefaultOptions, stream, block_begin, block_end);
}

extern "C" df11_status df11_decompress_chunked(const df11_header* hdr, const uint8_t* d_exp, const uint8_t* d_sm,
                                               const uint32_t* d_chunk_bit, const void* d_lut, uint16_t* d_out,
                                               uint32_t* d_status, void* stream) {
    df11_status st = check_header(hdr);
    if (st != DF11_OK) return st;
    if (hdr->n_elems == 0) return DF11_OK;
    if (!d_exp || !d_sm || !d_chunk_bit || !d_lut || !d_out)
        return fail(DF11_ERR_INVALID, "df11_decompress_chunked: null device pointer");
    if (!aligned16(d_exp) || !aligned16(d_sm) || !aligned16(d_chunk_bit) || !aligned16(d_lut) || !aligned16(d_out))
        return fail(DF11_ERR_INVALID, "df11_decompress_chunked: device pointers must be 16-byte aligned");
    if (hdr->total_bits >= (uint64_t(1) << 32))
        return fail(DF11_ERR_TOO_LARGE, "df11_decompress_chunked: chunk table positions are 32-bit");
    ChunkArgs a;
    a.exp32 = reinterpret_cast<const uint32_t*>(d_exp);
    a.sm8 = reinterpret_cast<const uint2*>(d_sm);
    a.chunk_bit = d_chunk_bit;
    a.lut = reinterpret_cast<const uint4*>(d_lut);
    a.out = d_out;
    a.status = d_status;
    a.n_elems = uint32_t(hdr->n_elems);
    a.n_chunks = uint32_t((hdr->n_elems + kIndChunk - 1) / kIndChunk);
    a.exp_words = uint32_t(hdr->bytes_exp / 4);
    constexpr size_t smem = kCompactBytes + size_t(kChunkWarps) * kChunkWarpBytes;
    static_assert(smem <= 227 * 1024, "shared memory per CTA");
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return fail(DF11_ERR_CUDA, "cudaGetDevice failed");
    LaunchInfo& li = g_info[dev][9];
    for (int attempt = 0;; attempt++) {
        if (!li.ready.load(std::memory_order_acquire)) {
            cudaError_t e = cudaFuncSetAttribute(decode_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 int(smem));
            if (e != cudaSuccess) return fail(DF11_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
            int sms = 0;
            e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return fail(DF11_ERR_CUDA, "SM count: %s", cudaGetErrorString(e));
            li.per_sm = 1;
            li.sms = sms;
            li.ready.store(1, std::memory_order_release);
        }
        const uint64_t groups = (uint64_t(a.n_chunks) + 31) / 32;
        const uint64_t want = (groups + kChunkWarps - 1) / kChunkWarps;
        const unsigned grid = unsigned(want < uint64_t(li.sms) ? want : uint64_t(li.sms));
        decode_chunk_kernel<<<grid, kChunkWarps * 32, smem, reinterpret_cast<cudaStream_t>(stream)>>>(a);
        const cudaError_t e = cudaGetLastError();
        if (e == cudaSuccess) break;
        if (attempt == 0) {  // a stale set-up (device reset, another context): redo it once
            li.ready.store(0, std::memory_order_release);
            continue;
        }
        return fail(DF11_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
    }
    return DF11_OK;
}

extern "C" df11_status df11_decode_kernel_info(const df11_header* hdr, uint32_t symbols_u8,
                                               const df11_decode_options* opt, df11_kernel_info* info) {
    if (!info) return fail(DF11_ERR_INVALID, "df11_decode_kernel_info: null info");
    df11_status st = check_header(hdr);
    if (st != DF11_OK) return st;
    Plan p;
    st = plan_for("df11_decode_kernel_info", hdr, symbols_u8 != 0, opt ? opt->peek_bits : 0, &p);
    if (st != DF11_OK) return st;
    Shape sh;
    st = shape_of(p, hdr->n_blocks, opt ? *opt : kDefaultOptions, &sh);
    if (st != DF11_OK) return st;
    std::memset(info, 0, sizeof(*info));
    std::snprintf(info->kernel, sizeof(info->kernel), "%s", p.name);
    info->grid = sh.grid;
    info->block = sh.block;
    info->smem_bytes = uint32_t(sh.smem);
    info->peek_bits = p.peek_bits;
    info->table_copies = p.copies;
    info->thread_blocks = hdr->n_blocks;
    return DF11_OK;
}
