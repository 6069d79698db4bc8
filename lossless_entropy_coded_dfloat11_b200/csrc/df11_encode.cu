// DF11 compression on the GPU: the exponent histogram (also per range of the
// encode grid), then, after the host has built the code, one encode kernel
// that finds each range's first stream bit and writes EncodedExponent,
// PackedSignMantissa, Gaps and the per-thread-block output positions.
//
// Format: "DFloat11: compressao sem perda para inferencia em GPU que reduz
// LLMs para 70% do tamanho", sections "O formato DFloat11" (Huffman-coded
// exponents, raw sign+mantissa bytes) and "Kernel de GPU em 2 etapas e
// metadados auxiliares" (8-byte thread windows, 5-bit gaps, one output
// position per thread block).
#include <cuda_runtime.h>

#include <atomic>
#include <chrono>
#include <cstring>
#include <type_traits>
#include <vector>

#include "df11_internal.h"

namespace df11 {

df11_status check_header(const df11_header* h);

namespace {

// Segments of the input, in elements of ES bytes: ES = 2 for BF16 weights
// (the symbol is the exponent field), ES = 1 for 8-bit symbols coded whole.
struct SegTable {
    const uint8_t* ptr[DF11_MAX_SEGMENTS];
    uint64_t start[DF11_MAX_SEGMENTS + 1];
    uint32_t n;
};

struct CodeTable {
    uint32_t code[256];
    uint8_t len[256];
};

// ---------------------------------------------------------------------------
// Histogram of the symbols of every segment in one launch (the exponent field
// of BF16 elements, or 8-bit symbols); per-warp shared-memory histograms.
// CTA r counts elements [r E, (r + 1) E) of the concatenated segments -- the
// elements of the encode kernel's range r -- and stores that range's
// histogram (32-bit counts) besides adding it to the 64-bit global counters;
// the encode kernel then needs no pass over its range to learn the range's
// code bits.  Within each segment's part of the range the threads read
// 16-byte vectors, four in flight per thread, and the unaligned ends element
// by element.
// ---------------------------------------------------------------------------
constexpr int kHistThreads = 256;

// Which plan left the per-range histograms in a workspace, and for which
// partition (written by the histogram kernel, checked by the encode kernel).
struct RangeTag {
    uint32_t token;     // the plan's token (never 0), also in df11_header.plan_token
    uint32_t n_ranges;
    uint64_t range_chunks;
};

template <int ES>
__device__ __forceinline__ void count16(uint32_t* mine, const uint4 q) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int k = 0; k < 4; k++) {
        if constexpr (ES == 2) {
            atomicAdd(&mine[(w[k] >> 7) & 0xFFu], 1u);
            atomicAdd(&mine[(w[k] >> 23) & 0xFFu], 1u);
        } else {
#pragma unroll
            for (int b = 0; b < 4; b++) atomicAdd(&mine[(w[k] >> (8 * b)) & 0xFFu], 1u);
        }
    }
}

template <int ES>
__device__ __forceinline__ uint32_t symbol_at(const uint8_t* p, uint64_t i) {
    if constexpr (ES == 2) return uint32_t(reinterpret_cast<const uint16_t*>(p)[i] >> 7) & 0xFFu;
    else return uint32_t(p[i]);
}

template <int ES>
__global__ void __launch_bounds__(kHistThreads) histogram_kernel(const __grid_constant__ SegTable sg,
                                                                 uint64_t range_elems,
                                                                 unsigned long long* __restrict__ hist,
                                                                 uint32_t* __restrict__ range_hist,
                                                                 RangeTag* __restrict__ tag, const RangeTag tag_value) {
    __shared__ uint32_t sh[kHistThreads / 32][256];
    uint32_t* mine = sh[threadIdx.x >> 5];
    for (int i = threadIdx.x; i < (kHistThreads / 32) * 256; i += kHistThreads) (&sh[0][0])[i] = 0;
    __syncthreads();
    const uint64_t n = sg.start[sg.n];
    const uint64_t e0 = uint64_t(blockIdx.x) * range_elems;
    const uint64_t e1 = e0 + range_elems < n ? e0 + range_elems : n;
    constexpr uint64_t kPerVec = 16 / ES;
    for (uint32_t seg = 0; seg < sg.n; seg++) {
        const uint64_t s0 = sg.start[seg], s1 = sg.start[seg + 1];
        if (s1 <= e0 || s0 >= e1) continue;
        // this range's part of the segment, local element indices [a, b)
        const uint64_t a = (e0 > s0 ? e0 : s0) - s0, b = (e1 < s1 ? e1 : s1) - s0;
        const uint8_t* p = sg.ptr[seg];  // 16-byte aligned
        uint64_t va = (a + kPerVec - 1) / kPerVec, vb = b / kPerVec;
        if (va > vb) va = vb = 0;  // no whole vector: every element below goes one by one
        const uint64_t h1 = va < vb ? va * kPerVec : b;  // scalar head [a, h1), tail [t0, b)
        const uint64_t t0 = va < vb ? vb * kPerVec : b;
        for (uint64_t i = a + threadIdx.x; i < h1; i += kHistThreads) atomicAdd(&mine[symbol_at<ES>(p, i)], 1u);
        for (uint64_t i = t0 + threadIdx.x; i < b; i += kHistThreads) atomicAdd(&mine[symbol_at<ES>(p, i)], 1u);
        const uint4* xv = reinterpret_cast<const uint4*>(p);
        uint64_t v = va + threadIdx.x;
        for (; v + 3 * kHistThreads < vb; v += 4 * kHistThreads) {
            uint4 x[4];
#pragma unroll
            for (int k = 0; k < 4; k++) x[k] = __ldcs(xv + v + k * kHistThreads);
#pragma unroll
            for (int k = 0; k < 4; k++) count16<ES>(mine, x[k]);
        }
        for (; v < vb; v += kHistThreads) count16<ES>(mine, __ldcs(xv + v));
    }
    __syncthreads();
    for (int s = threadIdx.x; s < 256; s += kHistThreads) {
        uint32_t t = 0;
        for (int w = 0; w < kHistThreads / 32; w++) t += sh[w][s];
        range_hist[uint64_t(blockIdx.x) * 256 + s] = t;
        if (t) atomicAdd(hist + s, (unsigned long long)t);
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) *tag = tag_value;
}

// Element i of the concatenated segments.
template <int ES>
__device__ __forceinline__ uint16_t load_elem(const SegTable& sg, uint64_t i, uint32_t& seg) {
    while (seg + 1 < sg.n && i >= sg.start[seg + 1]) seg++;
    const uint64_t rel = i - sg.start[seg];
    if constexpr (ES == 2) return reinterpret_cast<const uint16_t*>(sg.ptr[seg])[rel];
    else return sg.ptr[seg][rel];
}

__device__ __forceinline__ uint32_t find_seg(const SegTable& sg, uint64_t i) {
    uint32_t lo = 0, hi = sg.n - 1;
    while (lo < hi) {
        const uint32_t mid = (lo + hi + 1) >> 1;
        if (sg.start[mid] <= i) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// The kEncPerThread elements of this thread gathered one by one (those past
// n read as 0): threads whose elements straddle segments or are unaligned.
template <int ES>
__device__ __forceinline__ void load_chunk(const SegTable& sg, uint64_t i0, uint64_t n,
                                           uint16_t (&x)[kEncPerThread]) {
    uint32_t seg = find_seg(sg, i0 < n ? i0 : n - 1);
#pragma unroll
    for (int k = 0; k < int(kEncPerThread); k++) {
        const uint64_t i = i0 + k;
        x[k] = i < n ? load_elem<ES>(sg, i, seg) : uint16_t(0);
    }
}

// Block-wide exclusive scan of one value per thread; also returns the total.
template <int NT>
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* s_warp, uint32_t& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += y;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    uint32_t before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; w++) {
        const uint32_t t = s_warp[w];
        tot += t;
        before += (w < warp) ? t : 0u;
    }
    total = tot;
    return before + incl - v;
}

// ---------------------------------------------------------------------------
// The encode kernels are persistent: each CTA stages the code table in shared
// memory once and then walks chunks of kEncChunk elements in grid-stride
// order, loading the next chunk's elements while it works on the current one.
// (Indexing the table in the kernel's parameter space with a different
// exponent in every lane would serialise in the constant cache.)
// ---------------------------------------------------------------------------
struct SharedCodes {
    uint2 e[256];  // x = the code, right-aligned; y = its length (0 = absent)
};

__device__ __forceinline__ void stage_codes(SharedCodes& sc, const CodeTable& ct) {
    for (int v = threadIdx.x; v < 256; v += blockDim.x) sc.e[v] = make_uint2(ct.len[v] ? ct.code[v] : 0u, ct.len[v]);
}

// One thread's kEncPerThread elements packed in words (ES = 2: element 2j
// in the low half of word j; ES = 1: element 4j + q in byte q of word j),
// loaded ahead of use: 16 ES aligned bytes when they lie in one segment,
// else gathered element by element when used.
template <int ES>
constexpr int kWords = int(kEncPerThread) * ES / 4;

struct RawElems {
    uint4 a, b;  // b unused when ES = 1
    bool direct;
};

// c0 = the chunk's first element: its segment is looked up once (the same
// for every thread), a thread whose elements lie in a later segment looks
// up its own.
template <int ES>
__device__ __forceinline__ RawElems load_raw(const SegTable& sg, uint64_t c0, uint64_t i0, uint64_t n,
                                             uint32_t seg_hint = 0xFFFFFFFFu) {
    RawElems r;
    r.direct = false;
    if (i0 < n) {
        // the chunk's segment (given, or looked up); threads past its end
        // look up their own
        uint32_t seg = seg_hint != 0xFFFFFFFFu ? seg_hint : find_seg(sg, c0);
        if (i0 >= sg.start[seg + 1]) seg = find_seg(sg, i0);
        const uint8_t* p = sg.ptr[seg] + ES * (i0 - sg.start[seg]);
        if (i0 + kEncPerThread <= sg.start[seg + 1] && (reinterpret_cast<uintptr_t>(p) & 15u) == 0) {
            r.a = __ldcs(reinterpret_cast<const uint4*>(p));
            if constexpr (ES == 2) r.b = __ldcs(reinterpret_cast<const uint4*>(p) + 1);
            r.direct = true;
        }
    }
    return r;
}

template <int ES>
__device__ __forceinline__ void raw_words(const SegTable& sg, const RawElems& r, uint64_t i0, uint64_t n,
                                          uint32_t (&w)[kWords<ES>]) {
    if (r.direct) {
        w[0] = r.a.x; w[1] = r.a.y; w[2] = r.a.z; w[3] = r.a.w;
        if constexpr (ES == 2) {
            w[4] = r.b.x; w[5] = r.b.y; w[6] = r.b.z; w[7] = r.b.w;
        }
    } else {
        uint16_t x[kEncPerThread];
        load_chunk<ES>(sg, i0, n, x);
#pragma unroll
        for (int j = 0; j < kWords<ES>; j++) {
            if constexpr (ES == 2)
                w[j] = x[2 * j] | (uint32_t(x[2 * j + 1]) << 16);
            else
                w[j] = x[4 * j] | (uint32_t(x[4 * j + 1]) << 8) | (uint32_t(x[4 * j + 2]) << 16) |
                       (uint32_t(x[4 * j + 3]) << 24);
        }
    }
}

// The symbol of element k: the exponent field of a BF16 element, or the byte.
template <int ES>
__device__ __forceinline__ uint32_t symbol(const uint32_t (&w)[kWords<ES>], int k) {
    if constexpr (ES == 2) return (w[k >> 1] >> (16 * (k & 1) + 7)) & 0xFFu;
    else return (w[k >> 2] >> (8 * (k & 3))) & 0xFFu;
}

// Code bits of this thread's elements (those past n count 0).
template <int ES>
__device__ __forceinline__ uint32_t thread_bits(const SharedCodes& sc, const uint32_t (&w)[kWords<ES>],
                                                uint32_t valid) {
    uint32_t bits = 0;
    if (valid == kEncPerThread) {
#pragma unroll
        for (int k = 0; k < int(kEncPerThread); k++) bits += sc.e[symbol<ES>(w, k)].y;
    } else {
#pragma unroll
        for (int k = 0; k < int(kEncPerThread); k++)
            if (uint32_t(k) < valid) bits += sc.e[symbol<ES>(w, k)].y;
    }
    return bits;
}

// ---------------------------------------------------------------------------
// Encode: one persistent grid; CTA r (by an atomic ticket, so that every
// lower ticket's CTA is already running) takes a contiguous range of chunks
// of kEncChunk elements, 16 per thread.
//   the range's code bits: the dot product of the range's histogram (left
//     by the plan's histogram kernel) with the code lengths, or, without
//     that histogram, a first pass summing every element's code length;
//   look-back: the range's first stream bit by a decoupled look-back over
//     per-range descriptors (64 bits: a 2-bit state, then a bit count): the
//     CTA publishes its total as an "aggregate", walks back over its
//     predecessors adding aggregates until it meets an "inclusive" prefix, and
//     publishes its own inclusive prefix.  A predecessor holds an earlier
//     ticket, so it is running and publishes its aggregate without waiting on
//     anything; every wait is bounded anyway (after kSpinLimit polls the
//     range gives up and raises an abort flag, which marks the stream's
//     decode tables invalid once they are uploaded -- the decoders then
//     report the stream as corrupt);
//   pack: chunk by chunk, each thread's bit offset by a CTA scan, and the
//     chunk packed at the running prefix.
//
// Packing a chunk that starts at stream bit S.  Every code goes to its bit
// position in EncodedExponent (MSB first): each thread looks its 16 codes up
// once, appending them to a register row (2 words for BF16, 4 for 8-bit
// symbols), and after the CTA scan ORs the row into the (cleared) global
// array with one reduction per word it touches; a thread whose row
// overflowed ORs its codes one by one.  Words shared with neighbouring
// threads, chunks or ranges need no other care.  The same pass writes the
// sign+mantissa bytes, the gaps and the thread blocks' output positions:
//   * a code that starts inside window w-1 and runs into window w sets
//     gap[w] = s + l - 64w (s its start bit, l its length; gaps of windows
//     that begin exactly at a code start stay 0), OR-ed into the (cleared)
//     Gaps array;
//   * a code that starts exactly at bit 64*T*b sets off[b] = i, one that runs
//     over that bit sets off[b] = i + 1.
// Positions are kept 32-bit relative to S rounded down to a thread-block
// boundary; the code covering each window boundary in a thread's bits is
// found by a binary search over its codes' starts.
// ---------------------------------------------------------------------------
// Words in a thread's register row of codes: 16 exponent codes of ~2.6 bits
// fit 64 bits, 16 codes of 8-bit symbols (~7 bits for quantized weights) 128.
template <int ES>
constexpr int kRowWords = ES == 2 ? 2 : 4;
constexpr unsigned long long kDescAggregate = 1ull << 62, kDescInclusive = 2ull << 62;
constexpr unsigned long long kDescValue = (1ull << 62) - 1;
constexpr uint32_t kSpinLimit = 1u << 20;

// A descriptor is read only for its own value (no other memory is ordered by
// it), so relaxed GPU-scope accesses suffice: no fence, which would make every
// poll wait for the lane's outstanding pack stores.  Aligned 64-bit accesses
// are single-copy atomic.
__device__ __forceinline__ void publish(unsigned long long* p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long observe(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Warp 0: the exclusive prefix (first bit) of chunk c, whose own bits are
// `total`; publishes c's aggregate first and its inclusive prefix last.  The
// warp reads its predecessors kLookBack at a time (lane l, round r: the
// (l + 32 r)-th nearest), every load of a window in flight at once: with a
// few hundred chunks in flight, most look-backs end within one or two windows.
constexpr int kLookRounds = 4;
constexpr int kLookBack = 32 * kLookRounds;

__device__ __forceinline__ unsigned long long look_back(unsigned long long* desc, uint32_t c, uint32_t total,
                                                        uint32_t* abort_flag) {
    const uint32_t lane = threadIdx.x & 31u;
    if (c == 0) {
        if (lane == 0) publish(desc, kDescInclusive | total);
        return 0;
    }
    if (lane == 0) publish(desc + c, kDescAggregate | total);
    unsigned long long prefix = 0;
    int64_t base = int64_t(c) - 1;  // the nearest predecessor not yet added
    uint32_t spins = 0;
    for (;;) {
        unsigned long long d[kLookRounds];
#pragma unroll
        for (int r = 0; r < kLookRounds; r++) {
            const int64_t j = base - int64_t(lane) - 32 * r;
            d[r] = j >= 0 ? observe(desc + j) : kDescInclusive;
        }
        // walk the window nearest first; stop at the first inclusive prefix
        bool stall = false, found = false;
        unsigned long long v = 0;
#pragma unroll
        for (int r = 0; r < kLookRounds; r++) {
            const uint32_t state = uint32_t(d[r] >> 62);
            const uint32_t incl = __ballot_sync(0xFFFFFFFFu, state == 2u);
            const uint32_t empty = __ballot_sync(0xFFFFFFFFu, state == 0u);
            // lanes up to the nearest inclusive prefix (all 32 if none) must be ready
            const uint32_t upto = incl ? (incl & (0u - incl)) * 2u - 1u : 0xFFFFFFFFu;
            if (empty & upto) {
                stall = true;
                break;
            }
            v += ((upto >> lane) & 1u) ? (d[r] & kDescValue) : 0ull;
            if (incl) {
                found = true;
                break;
            }
        }
        if (stall) {
            ++spins;
            // never expected: give up and raise the abort flag (the stream
            // is then marked bad, mark_if_aborted); once one range has
            // given up, the others stop waiting too
            const bool abort = spins >= kSpinLimit ||
                               ((spins & 63u) == 0 && *reinterpret_cast<volatile uint32_t*>(abort_flag) != 0u);
            if (abort) {
                if (lane == 0) atomicExch(abort_flag, 1u);
                return prefix;
            }
            __nanosleep(32);
            continue;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
        prefix += v;
        if (found) break;
        base -= kLookBack;
    }
    if (lane == 0) publish(desc + c, kDescInclusive | (prefix + total));
    return prefix;
}

template <int ES>
__global__ void __launch_bounds__(kEncThreads, 4) encode_kernel(const __grid_constant__ SegTable sg,
                                                             const __grid_constant__ CodeTable ct, uint64_t n,
                                                             uint64_t n_chunks, uint64_t chunks_per_range,
                                                             uint32_t log2_block_bits,
                                                             unsigned long long* __restrict__ desc,
                                                             uint32_t* __restrict__ ticket, uint32_t* abort_flag,
                                                             uint32_t* __restrict__ exp32, uint8_t* __restrict__ sm,
                                                             uint32_t* __restrict__ gaps32,
                                                             uint32_t* __restrict__ block_off, uint64_t n_blocks,
                                                             uint32_t* __restrict__ chunk_bit,
                                                             const uint32_t* __restrict__ range_hist,
                                                             const RangeTag* __restrict__ tag, const RangeTag expect) {
    __shared__ SharedCodes sc;
    // per element: its code's start relative to its thread's first bit
    __shared__ uint32_t s_pos[kEncPerThread][kEncThreads];
    __shared__ uint32_t s_warp[2][kEncThreads / 32];  // scan partials, two chunks apart
    __shared__ uint32_t s_ticket;
    __shared__ unsigned long long s_prefix;
    stage_codes(sc, ct);
    if (threadIdx.x == 0) s_ticket = atomicAdd(ticket, 1u);
    __syncthreads();
    const uint64_t block_mask = (uint64_t(1) << log2_block_bits) - 1;
    const uint64_t tofs = uint64_t(threadIdx.x) * kEncPerThread;
    const uint32_t range = s_ticket;
    const uint64_t c_begin = uint64_t(range) * chunks_per_range;
    const uint64_t c_end = c_begin + chunks_per_range < n_chunks ? c_begin + chunks_per_range : n_chunks;
    if (c_begin >= c_end) return;  // (the grid has exactly one range per CTA)

    // the segment holding a chunk's first element, advanced chunk by chunk
    auto seg_of = [&](uint32_t seg, uint64_t c) {
        while (seg + 1 < sg.n && c * kEncChunk >= sg.start[seg + 1]) seg++;
        return seg;
    };
    const uint32_t seg0 = find_seg(sg, c_begin * kEncChunk);

    // the code bits of this range: from the plan's histogram of the range
    // when the workspace holds this partition's (thread s: symbol s), else
    // a first pass reads the range once for the sum
    uint32_t mine = 0;
    bool from_hist = false;
    if (expect.token != 0) {
        const RangeTag have = *tag;
        from_hist = have.token == expect.token && have.n_ranges == expect.n_ranges &&
                    have.range_chunks == expect.range_chunks;
    }
    if (from_hist) {
        static_assert(kEncThreads == 256, "one thread per symbol");
        mine = range_hist[uint64_t(range) * 256 + threadIdx.x] * sc.e[threadIdx.x].y;
    } else {
        uint32_t seg = seg0;
        RawElems next = load_raw<ES>(sg, c_begin * kEncChunk, c_begin * kEncChunk + tofs, n, seg);
        for (uint64_t c = c_begin; c < c_end; c++) {
            const RawElems cur = next;
            if (c + 1 < c_end) {
                seg = seg_of(seg, c + 1);
                next = load_raw<ES>(sg, (c + 1) * kEncChunk, (c + 1) * kEncChunk + tofs, n, seg);
            }
            const uint64_t i0 = c * kEncChunk + tofs;
            if (i0 < n) {
                uint32_t w8[kWords<ES>];
                raw_words<ES>(sg, cur, i0, n, w8);
                const uint64_t left = n - i0;
                mine += thread_bits<ES>(sc, w8, left < kEncPerThread ? uint32_t(left) : kEncPerThread);
            }
        }
    }
    // the pack's first loads go out before the look-back
    uint32_t seg = seg0;
    RawElems next = load_raw<ES>(sg, c_begin * kEncChunk, c_begin * kEncChunk + tofs, n, seg);
    uint32_t range_total;
    block_exclusive_scan<kEncThreads>(mine, s_warp[0], range_total);
    // the range's first bit: one look-back per range; every earlier range's
    // CTA is already running (it holds an earlier ticket) and publishes its
    // aggregate as soon as it has its range's bits
    if (threadIdx.x < 32) {
        const unsigned long long pre = look_back(desc, range, range_total, abort_flag);
        if (threadIdx.x == 0) s_prefix = pre;
    }
    __syncthreads();
    uint64_t S = s_prefix;

    // pack: each chunk at the running prefix.  No barrier at the top of the
    // loop: s_pos is the thread's own column, and the scan alternates between
    // two s_warp rows (a warp writes a row again only after every warp has
    // passed the scan in between).
    for (uint64_t c = c_begin; c < c_end; c++) {
        const RawElems cur = next;
        if (c + 1 < c_end) {
            seg = seg_of(seg, c + 1);
            next = load_raw<ES>(sg, (c + 1) * kEncChunk, (c + 1) * kEncChunk + tofs, n, seg);
        }
        const uint64_t i0 = c * kEncChunk + tofs;
        uint32_t w8[kWords<ES>];
        uint32_t valid = 0, bits = 0;
        // the thread's codes in a row, right-aligned: x[0] holds the last bits
        uint32_t x[kRowWords<ES>];
#pragma unroll
        for (int j = 0; j < kRowWords<ES>; j++) x[j] = 0;
        if (i0 < n) {
            raw_words<ES>(sg, cur, i0, n, w8);
            const uint64_t left = n - i0;
            valid = left < kEncPerThread ? uint32_t(left) : kEncPerThread;
            // one lookup per code: its start relative to the thread's first
            // bit to s_pos, the code appended to the row
            auto gather = [&](auto full_tag) {
                constexpr bool kFull = decltype(full_tag)::value;
#pragma unroll
                for (int k = 0; k < int(kEncPerThread); k++) {
                    // code (right-aligned) and length; 0, 0 past the valid elements
                    const uint2 e = (kFull || uint32_t(k) < valid) ? sc.e[symbol<ES>(w8, k)] : make_uint2(0, 0);
                    s_pos[k][threadIdx.x] = bits;
#pragma unroll
                    for (int j = kRowWords<ES> - 1; j > 0; j--) x[j] = __funnelshift_lc(x[j - 1], x[j], e.y);
                    x[0] = __funnelshift_lc(0u, x[0], e.y) | e.x;
                    bits += e.y;
                }
            };
            if (valid == kEncPerThread)
                gather(std::true_type{});
            else
                gather(std::false_type{});
        }
        uint32_t chunk_total;
        const uint32_t my_off =
            block_exclusive_scan<kEncThreads>(bits, s_warp[uint32_t(c - c_begin) & 1u], chunk_total);
        const uint32_t lead = uint32_t(S & 31u);
        const uint64_t Sb = S & ~block_mask;  // a thread-block (and window) boundary
        // gap fields of this chunk: windows (S >> 6, (S + total - 1) >> 6], at
        // gap array bits 5w .. 5w + 4, from gap array word g0 on
        const uint64_t g0 = (5 * ((S >> 6) + 1)) >> 5;
        const uint64_t blk_base = Sb >> log2_block_bits;
        // gap array bit 5w of window w = Sb / 64 + j, counted from word g0's
        // first bit: gap_bit0 + 5 j (small: Sb is at most one thread block,
        // 64 T bits, before the chunk's first window)
        const int32_t gap_bit0 = int32_t(int64_t(5 * (Sb >> 6)) - int64_t(32 * g0));
        // Word wi of the chunk's bits (counted from S rounded down to a word),
        // MSB first, OR-ed into the (cleared) EncodedExponent: words shared
        // with neighbouring threads, chunks or ranges need no other care.
        auto or_word = [&](uint32_t wi, uint32_t v) {
            if (v) atomicOr(exp32 + (S >> 5) + wi, __byte_perm(v, 0, 0x0123));
        };
        if (valid) {
            const uint32_t pos = lead + my_off;  // from S rounded down to a word
            if (bits <= 32u * kRowWords<ES>) {
                // the whole row at once: with the row's end at bit e, the word
                // k places before e's word holds row words k and k-1 shifted
                // by 32 - e % 32 (no shift when e is word-aligned)
                if (bits) {
                    const uint32_t e = pos + bits, sh = 32u - (e & 31u), wl = (e - 1) >> 5;
                    or_word(wl, __funnelshift_l(0u, x[0], sh));
#pragma unroll
                    for (int k = 1; k < kRowWords<ES>; k++)
                        if (uint32_t(k) <= wl) or_word(wl - k, __funnelshift_l(x[k - 1], x[k], sh));
                    if (uint32_t(kRowWords<ES>) <= wl)
                        or_word(wl - kRowWords<ES>, __funnelshift_l(x[kRowWords<ES> - 1], 0u, sh));
                }
            } else {  // rare: the row overflowed; code by code
                uint32_t p = pos;
                auto pack = [&](auto full_tag) {
                    constexpr bool kFull = decltype(full_tag)::value;
#pragma unroll
                    for (int k = 0; k < int(kEncPerThread); k++) {
                        const uint2 e = (kFull || uint32_t(k) < valid) ? sc.e[symbol<ES>(w8, k)] : make_uint2(0, 0);
                        const uint32_t t = __funnelshift_l(0u, e.x, 32u - e.y);  // left-aligned (l = 32: shift 0)
                        or_word(p >> 5, t >> (p & 31u));
                        or_word((p >> 5) + 1, __funnelshift_r(0u, t, p & 31u));  // the bits that did not fit
                        p += e.y;
                    }
                };
                if (valid == kEncPerThread)
                    pack(std::true_type{});
                else
                    pack(std::false_type{});
            }
            if (gaps32) {
                // every window boundary in the thread's bits [A, A + bits)
                // (A relative to Sb), at q from the thread's first bit, is
                // covered by one code: the last one starting at or before it
                // (binary search over the thread's starts; starts past the
                // valid elements equal bits).  If that code starts before the
                // boundary, the window's gap is where the next code starts (the
                // gaps of windows that begin with a code stay 0); at a
                // thread-block boundary the block's first element is that
                // code's, or the next one's.
                const uint32_t A = uint32_t(S - Sb) + my_off;
                uint32_t* const gap_words = gaps32 + g0;
                for (uint32_t q = (64u - (A & 63u)) & 63u; q < bits; q += 64) {
                    uint32_t k = 0;
                    if (s_pos[k + 8][threadIdx.x] <= q) k += 8;
                    if (s_pos[k + 4][threadIdx.x] <= q) k += 4;
                    if (s_pos[k + 2][threadIdx.x] <= q) k += 2;
                    if (s_pos[k + 1][threadIdx.x] <= q) k += 1;
                    const bool inside = s_pos[k][threadIdx.x] < q;  // the code starts before the boundary
                    const uint32_t Bq = A + q;                       // the boundary, from Sb
                    if (inside) {
                        const uint32_t b = k + 1 < kEncPerThread ? s_pos[k + 1][threadIdx.x] : bits;
                        const uint32_t gb = uint32_t(gap_bit0 + int32_t(5 * (Bq >> 6)));
                        const uint32_t sh = gb & 31u, g = b - q;
                        atomicOr(gap_words + (gb >> 5), g << sh);
                        if (sh > 27) atomicOr(gap_words + (gb >> 5) + 1, g >> (32 - sh));
                    }
                    if ((Bq & uint32_t(block_mask)) == 0)
                        block_off[blk_base + (Bq >> log2_block_bits)] = uint32_t(i0) + k + (inside ? 1u : 0u);
                }
            }
        }
        if (block_off && valid && n - i0 <= kEncPerThread) block_off[n_blocks] = uint32_t(n);
        if (chunk_bit && valid) {  // independent-chunk table: first bit of every kIndChunk elements
            if (i0 % kIndChunk == 0) chunk_bit[i0 / kIndChunk] = uint32_t(S + my_off);
            if (n - i0 <= kEncPerThread) chunk_bit[(n + kIndChunk - 1) / kIndChunk] = uint32_t(S + my_off + bits);
        }
        if constexpr (ES == 2) if (valid) {
            // sign+mantissa bytes: sign (bit 15) to bit 7, mantissa bits 6..0
            uint32_t smw[kEncPerThread / 4];
#pragma unroll
            for (int j = 0; j < int(kEncPerThread / 4); j++) {
                const uint32_t a = w8[2 * j], b = w8[2 * j + 1];
                const uint32_t pa = ((a >> 8) & 0x00800080u) | (a & 0x007F007Fu);  // bytes 0 and 2
                const uint32_t pb = ((b >> 8) & 0x00800080u) | (b & 0x007F007Fu);
                smw[j] = __byte_perm(pa, pb, 0x6420);
            }
            if (valid == kEncPerThread) {
                __stcs(reinterpret_cast<uint4*>(sm + i0), make_uint4(smw[0], smw[1], smw[2], smw[3]));
            } else {
#pragma unroll
                for (int k = 0; k < int(kEncPerThread); k++)
                    if (uint32_t(k) < valid) sm[i0 + k] = uint8_t(smw[k >> 2] >> (8 * (k & 3)));
            }
        }
        S += chunk_total;
    }
}

// After the decode tables' upload: a stream whose encode gave up (see
// look_back) gets a zero table magic, so that every decode of it fails.
__global__ void mark_if_aborted(const uint32_t* abort_flag, uint32_t* lut_magic) {
    if (*abort_flag) *lut_magic = 0u;
}

// Persistent grid for an encode kernel: as many CTAs as can be resident on
// every SM at once.
// (SMs × resident CTAs per SM, looked up once per device and kernel: the plan
// and the encode of every compress call ask again.)
constexpr int kMaxDevices = 64;
template <int ES>
unsigned encode_grid(uint64_t chunks) {
    static std::atomic<uint32_t> cached[kMaxDevices];  // 0 = not yet
    int dev = 0;
    cudaGetDevice(&dev);
    uint32_t slots = dev >= 0 && dev < kMaxDevices ? cached[dev].load(std::memory_order_relaxed) : 0u;
    if (!slots) {
        int sms = 148, per_sm = 1;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, encode_kernel<ES>, kEncThreads, 0) != cudaSuccess ||
            per_sm < 1)
            per_sm = 1;
        slots = uint32_t(sms) * uint32_t(per_sm);
        if (dev >= 0 && dev < kMaxDevices) cached[dev].store(slots, std::memory_order_relaxed);
    }
    uint64_t want = slots;
    if (want > kMaxEncRanges) want = kMaxEncRanges;
    return unsigned(chunks < want ? chunks : want);
}

// The encode kernel's partition of `chunks` chunks: one contiguous range of
// range_chunks chunks per CTA of a full persistent grid (the last range may
// be shorter).  The plan's histogram kernel counts by the same ranges.
template <int ES>
RangeTag encode_partition(uint64_t chunks) {
    RangeTag t{0u, 0u, 0u};
    if (!chunks) return t;
    const uint64_t slots = encode_grid<ES>(chunks);
    t.range_chunks = (chunks + slots - 1) / slots;
    t.n_ranges = uint32_t((chunks + t.range_chunks - 1) / t.range_chunks);
    return t;
}

// A fresh nonzero token per plan (an odd stride visits every 32-bit value).
uint32_t next_plan_token() {
    static std::atomic<uint32_t> counter{
        uint32_t(std::chrono::steady_clock::now().time_since_epoch().count()) | 1u};
    uint32_t t;
    do t = counter.fetch_add(0x9E3779B9u); while (t == 0);
    return t;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Encode scratch: one look-back descriptor per chunk, then the chunk ticket
// and the abort flag, 8 bytes each (zeroed by every encode call before its
// kernel).
constexpr uint64_t encode_scratch_bytes(uint64_t chunks) { return 8 * (chunks + 2); }

struct Workspace {
    unsigned long long* hist;
    RangeTag* tag;
    unsigned long long* desc;
    uint32_t* range_hist;
};

df11_status carve(void* ws, uint64_t ws_bytes, uint64_t n_elems, Workspace* w) {
    uint64_t need = 0;
    df11_compress_workspace_size(n_elems, &need);
    if (!ws) return fail(DF11_ERR_INVALID, "null workspace");
    if (!aligned16(ws)) return fail(DF11_ERR_INVALID, "workspace must be 16-byte aligned");
    if (ws_bytes < need)
        return fail(DF11_ERR_CAPACITY, "workspace of %llu bytes, need %llu", (unsigned long long)ws_bytes,
                    (unsigned long long)need);
    const uint64_t chunks = (n_elems + kEncChunk - 1) / kEncChunk;
    uint8_t* p = static_cast<uint8_t*>(ws);
    w->hist = reinterpret_cast<unsigned long long*>(p);
    w->tag = reinterpret_cast<RangeTag*>(p + kWsTagOff);
    w->desc = reinterpret_cast<unsigned long long*>(p + kWsDescOff);
    w->range_hist = reinterpret_cast<uint32_t*>(p + ws_range_hist_off(chunks));
    return DF11_OK;
}

df11_status cuda_fail(const char* what, cudaError_t e) {
    return fail(DF11_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

df11_status build_segtable(const void* const* d_segs, const uint64_t* counts, uint32_t n_segs, SegTable* sg,
                           uint64_t* n_total) {
    if (!d_segs || !counts) return fail(DF11_ERR_INVALID, "null segment arrays");
    if (n_segs < 1 || n_segs > DF11_MAX_SEGMENTS)
        return fail(DF11_ERR_INVALID, "n_segs %u outside 1..%d", n_segs, DF11_MAX_SEGMENTS);
    std::memset(sg, 0, sizeof(*sg));
    uint64_t acc = 0;
    for (uint32_t k = 0; k < n_segs; k++) {
        if (counts[k] && !d_segs[k]) return fail(DF11_ERR_INVALID, "null segment %u", k);
        if (counts[k] && !aligned16(d_segs[k]))
            return fail(DF11_ERR_INVALID, "segment %u is not 16-byte aligned", k);
        sg->ptr[k] = static_cast<const uint8_t*>(d_segs[k]);
        sg->start[k] = acc;
        acc += counts[k];
    }
    sg->start[n_segs] = acc;
    sg->n = n_segs;
    if (acc >= (uint64_t(1) << 32)) return fail(DF11_ERR_TOO_LARGE, "more than 2^32 - 1 elements");
    *n_total = acc;
    return DF11_OK;
}

// Histogram kernel (one launch; a histogram per encode range too), host code
// builder, header.
template <int ES>
df11_status compress_plan(const void* const* d_segs, const uint64_t* seg_counts, uint32_t n_segs,
                          uint32_t threads_per_block, uint32_t max_code_len, void* d_workspace,
                          uint64_t workspace_bytes, df11_header* hdr, void* stream) {
    if (!hdr) return fail(DF11_ERR_INVALID, "null header");
    SegTable sg;
    uint64_t n = 0;
    df11_status st = build_segtable(d_segs, seg_counts, n_segs, &sg, &n);
    if (st != DF11_OK) return st;
    Workspace w{};
    st = carve(d_workspace, workspace_bytes, n, &w);
    if (st != DF11_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(w.hist, 0, 2048, s);
    if (e != cudaSuccess) return cuda_fail("histogram clear", e);
    uint32_t token = 0;
    if (n) {
        RangeTag tag = encode_partition<ES>((n + kEncChunk - 1) / kEncChunk);
        tag.token = token = next_plan_token();
        histogram_kernel<ES><<<tag.n_ranges, kHistThreads, 0, s>>>(sg, tag.range_chunks * kEncChunk, w.hist,
                                                                   w.range_hist, w.tag, tag);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("histogram launch", e);
    uint64_t hist[256];
    e = cudaMemcpyAsync(hist, w.hist, sizeof(hist), cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_fail("histogram readback", e);
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail("histogram sync", e);
    uint8_t len[256];
    st = df11_code_lengths(hist, max_code_len, len);
    if (st != DF11_OK) return st;
    uint64_t bits = 0;
    for (int v = 0; v < 256; v++) bits += hist[v] * len[v];
    st = df11_header_init(hdr, len, n, bits, threads_per_block, max_code_len, seg_counts, n_segs);
    if (st == DF11_OK) hdr->plan_token = token;
    return st;
}

// Clears and the encode kernel, then the decode tables: built on the host
// while the kernel runs, uploaded after it.
// d_sm is written for BF16 input (ES = 2) only.
// With d_chunk_bit (the independent-chunk table instead of Gaps and block
// offsets) d_gaps and d_block_off are not written and may be null.
template <int ES>
df11_status compress_encode(const char* fn, const void* const* d_segs, const df11_header* hdr,
                            unsigned long long* desc, const uint32_t* range_hist, const RangeTag* tag,
                            uint8_t* d_exp, uint8_t* d_sm,
                            uint8_t* d_gaps, uint32_t* d_block_off, void* d_lut, void* stream,
                            uint32_t* d_chunk_bit = nullptr) {
    df11_status st = check_header(hdr);
    if (st != DF11_OK) return st;
    uint64_t counts[DF11_MAX_SEGMENTS];
    if (hdr->n_segments < 1 || hdr->n_segments > DF11_MAX_SEGMENTS)
        return fail(DF11_ERR_INVALID, "header n_segments %u", hdr->n_segments);
    for (uint32_t k = 0; k < hdr->n_segments; k++) counts[k] = hdr->seg_elem_off[k + 1] - hdr->seg_elem_off[k];
    SegTable sg;
    uint64_t n = 0;
    st = build_segtable(d_segs, counts, hdr->n_segments, &sg, &n);
    if (st != DF11_OK) return st;
    if (n != hdr->n_elems) return fail(DF11_ERR_INVALID, "segments disagree with header n_elems");
    const bool chunked = d_chunk_bit != nullptr;
    if (!d_exp || (ES == 2 && !d_sm) || (!chunked && (!d_gaps || !d_block_off)) || !d_lut)
        return fail(DF11_ERR_INVALID, "%s: null output pointer", fn);
    if (!aligned16(d_exp) || (ES == 2 && !aligned16(d_sm)) || (!chunked && (!aligned16(d_gaps) ||
        !aligned16(d_block_off))) || !aligned16(d_lut))
        return fail(DF11_ERR_INVALID, "%s: outputs must be 16-byte aligned", fn);
    if (chunked && hdr->total_bits >= (uint64_t(1) << 32))
        return fail(DF11_ERR_TOO_LARGE, "%s: chunk table positions are 32-bit", fn);

    CodeTable ct;
    std::memcpy(ct.len, hdr->code_len, 256);
    if (!canonical_codes(hdr->code_len, ct.code)) return fail(DF11_ERR_INVALID, "code lengths overflow");

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if ((e = cudaMemsetAsync(d_exp, 0, hdr->bytes_exp, s)) != cudaSuccess) return cuda_fail("clear exp", e);
    if (!chunked) {
        if ((e = cudaMemsetAsync(d_gaps, 0, hdr->bytes_gaps, s)) != cudaSuccess) return cuda_fail("clear gaps", e);
        if ((e = cudaMemsetAsync(d_block_off, 0, hdr->bytes_off, s)) != cudaSuccess)
            return cuda_fail("clear off", e);
    }
    if constexpr (ES == 2) {
        const uint64_t sm_tail = n & ~uint64_t(15);
        if (hdr->bytes_sm > sm_tail &&
            (e = cudaMemsetAsync(d_sm + sm_tail, 0, hdr->bytes_sm - sm_tail, s)) != cudaSuccess)
            return cuda_fail("clear sm tail", e);
    }
    const uint64_t chunks = (n + kEncChunk - 1) / kEncChunk;
    if (chunks >= (uint64_t(1) << 31)) return fail(DF11_ERR_TOO_LARGE, "too many chunks");
    uint32_t* abort_flag = reinterpret_cast<uint32_t*>(desc + chunks + 1);
    if (n) {
        if ((e = cudaMemsetAsync(desc, 0, encode_scratch_bytes(chunks), s)) != cudaSuccess)
            return cuda_fail("clear encode scratch", e);
        uint32_t log2_bb = 6;
        while ((1u << (log2_bb - 6)) < hdr->threads_per_block) log2_bb++;
        // one contiguous range of chunks per CTA of a full persistent grid;
        // the plan's per-range histograms are used when the workspace holds
        // this header's plan for this partition (the kernel compares tags)
        RangeTag expect = encode_partition<ES>(chunks);
        expect.token = range_hist && tag ? hdr->plan_token : 0u;
        // a range's code bits are counted in 32 bits: at most 32 per element
        if (expect.range_chunks * kEncChunk * 32 >= (uint64_t(1) << 32))
            return fail(DF11_ERR_TOO_LARGE, "%s: %llu elements per encode range on this device", fn,
                        (unsigned long long)(expect.range_chunks * kEncChunk));
        encode_kernel<ES><<<expect.n_ranges, kEncThreads, 0, s>>>(
            sg, ct, n, chunks, expect.range_chunks, log2_bb, desc, reinterpret_cast<uint32_t*>(desc + chunks),
            abort_flag, reinterpret_cast<uint32_t*>(d_exp), d_sm, reinterpret_cast<uint32_t*>(d_gaps),
            d_block_off, hdr->n_blocks, d_chunk_bit, range_hist, tag, expect);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail("encode launch", e);
    }
    // The decode tables are built while the encode kernel runs, in this
    // thread's own host buffer (no heap; an asynchronous copy from pageable
    // memory has taken the bytes when it returns), and uploaded after it.
    static thread_local unsigned char lut[kLutBytes];
    st = df11_build_lut(hdr, lut, sizeof(lut));
    if (st != DF11_OK) return st;
    if ((e = cudaMemcpyAsync(d_lut, lut, kLutBytes, cudaMemcpyHostToDevice, s)) != cudaSuccess)
        return cuda_fail("table upload", e);
    if (n) {
        mark_if_aborted<<<1, 1, 0, s>>>(abort_flag, static_cast<uint32_t*>(d_lut));
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail("abort mark launch", e);
    }
    return DF11_OK;
}

}  // namespace
}  // namespace df11

using namespace df11;

extern "C" df11_status df11_compress_plan(const void* const* d_segs, const uint64_t* seg_counts, uint32_t n_segs,
                                          uint32_t threads_per_block, uint32_t max_code_len, void* d_workspace,
                                          uint64_t workspace_bytes, df11_header* hdr, void* stream) {
    return compress_plan<2>(d_segs, seg_counts, n_segs, threads_per_block, max_code_len, d_workspace,
                            workspace_bytes, hdr, stream);
}

extern "C" df11_status df11_compress_encode(const void* const* d_segs, const df11_header* hdr, void* d_workspace,
                                            uint64_t workspace_bytes, uint8_t* d_exp, uint8_t* d_sm,
                                            uint8_t* d_gaps, uint32_t* d_block_off, void* d_lut,
                                            void* stream) {
    Workspace w{};
    const df11_status st = carve(d_workspace, workspace_bytes, hdr ? hdr->n_elems : 0, &w);
    if (st != DF11_OK) return st;
    return compress_encode<2>("df11_compress_encode", d_segs, hdr, w.desc, w.range_hist, w.tag, d_exp, d_sm,
                              d_gaps, d_block_off, d_lut, stream);
}

extern "C" df11_status df11_compress_plan_u8(const void* const* d_segs, const uint64_t* seg_counts,
                                             uint32_t n_segs, uint32_t threads_per_block, uint32_t max_code_len,
                                             void* d_workspace, uint64_t workspace_bytes, df11_header* hdr,
                                             void* stream) {
    return compress_plan<1>(d_segs, seg_counts, n_segs, threads_per_block, max_code_len, d_workspace,
                            workspace_bytes, hdr, stream);
}

extern "C" df11_status df11_compress_encode_u8(const void* const* d_segs, const df11_header* hdr,
                                               void* d_workspace, uint64_t workspace_bytes, uint8_t* d_exp,
                                               uint8_t* d_gaps, uint32_t* d_block_off, void* d_lut,
                                               void* stream) {
    Workspace w{};
    const df11_status st = carve(d_workspace, workspace_bytes, hdr ? hdr->n_elems : 0, &w);
    if (st != DF11_OK) return st;
    return compress_encode<1>("df11_compress_encode_u8", d_segs, hdr, w.desc, w.range_hist, w.tag, d_exp,
                              nullptr, d_gaps, d_block_off, d_lut, stream);
}

// ---------------------------------------------------------------------------
// Encode without any allocation: the same kernels as df11_compress_encode,
// with their scratch (look-back descriptors, chunk ticket, abort flag) in a
// fixed-size array that lives in the library's own device memory.  For
// callers that cannot allocate device memory when they compress: serving
// engines that hand all of HBM to their own pools at start-up and forbid
// later cudaMalloc calls, and code running inside an allocator (an
// out-of-memory handler, say) where allocating would recurse.
// ---------------------------------------------------------------------------
namespace df11 {
namespace {

constexpr uint64_t kStaticChunks = DF11_STATIC_MAX_ELEMS / kEncChunk;
constexpr uint64_t kStaticScratchBytes = encode_scratch_bytes(kStaticChunks);
static_assert(DF11_STATIC_MAX_ELEMS % kEncChunk == 0, "whole chunks");

// Loaded with the library's device code on every GPU that uses it and held
// until exit.  Every call clears the part it uses (the look-back descriptors
// and the chunk ticket must start at zero) before its kernel; two calls that
// overlap on the GPU share it and race.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of the scratch for the current device and context.  Host
// code cannot use the symbol itself as a device pointer, and the address can
// change when the module is loaded again (after cudaDeviceReset, or in another
// context on the same device), so it is looked up on every call; once the
// library's device code is loaded, the lookup allocates nothing.
df11_status static_scratch_address(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail("cudaGetSymbolAddress(static scratch)", e);
    *out = p;
    return DF11_OK;
}

}  // namespace
}  // namespace df11

extern "C" df11_status df11_compress_encode_static(const void* const* d_segs, const df11_header* hdr,
                                                   uint8_t* d_exp, uint8_t* d_sm, uint8_t* d_gaps,
                                                   uint32_t* d_block_off, void* d_lut, void* stream) {
    df11_status st = check_header(hdr);
    if (st != DF11_OK) return st;
    if (hdr->n_elems > DF11_STATIC_MAX_ELEMS)
        return fail(DF11_ERR_TOO_LARGE,
                    "df11_compress_encode_static: %llu elements, its fixed scratch holds at most %llu; "
                    "use df11_compress_encode with a workspace",
                    (unsigned long long)hdr->n_elems, (unsigned long long)DF11_STATIC_MAX_ELEMS);
    void* scratch = nullptr;
    st = static_scratch_address(&scratch);
    if (st != DF11_OK) return st;
    return compress_encode<2>("df11_compress_encode_static", d_segs, hdr, static_cast<unsigned long long*>(scratch),
                              nullptr, nullptr, d_exp, d_sm,
                              d_gaps, d_block_off, d_lut, stream);
}

extern "C" df11_status df11_compress_encode_chunked(const void* const* d_segs, const df11_header* hdr,
                                                    void* d_workspace, uint64_t workspace_bytes, uint8_t* d_exp,
                                                    uint8_t* d_sm, uint32_t* d_chunk_bit, void* d_lut,
                                                    void* stream) {
    if (!d_chunk_bit || (reinterpret_cast<uintptr_t>(d_chunk_bit) & 15u))
        return fail(DF11_ERR_INVALID, "df11_compress_encode_chunked: chunk table null or not 16-byte aligned");
    Workspace w{};
    const df11_status st = carve(d_workspace, workspace_bytes, hdr ? hdr->n_elems : 0, &w);
    if (st != DF11_OK) return st;
    return compress_encode<2>("df11_compress_encode_chunked", d_segs, hdr, w.desc, w.range_hist, w.tag, d_exp,
                              d_sm, nullptr, nullptr, d_lut, stream, d_chunk_bit);
}
