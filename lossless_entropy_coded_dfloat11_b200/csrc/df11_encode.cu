// DF11 compression on the GPU: exponent histogram, then (after the host has
// built the code) per-chunk code-bit totals, their prefix sum, and the
// bit-pack kernel that writes EncodedExponent, PackedSignMantissa, Gaps and
// the per-thread-block output positions.
//
// Format: "DFloat11: compressao sem perda para inferencia em GPU que reduz
// LLMs para 70% do tamanho", sections "O formato DFloat11" (Huffman-coded
// exponents, raw sign+mantissa bytes) and "Kernel de GPU em 2 etapas e
// metadados auxiliares" (8-byte thread windows, 5-bit gaps, one output
// position per thread block).
#include <cuda_runtime.h>

#include <atomic>
#include <cstring>
#include <mutex>
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
// Histogram of the symbols of one segment (the exponent field of BF16
// elements, or 8-bit symbols); per-warp shared-memory histograms, flushed
// into 64-bit global counters.
// ---------------------------------------------------------------------------
constexpr int kHistThreads = 256;

__global__ void __launch_bounds__(kHistThreads) histogram_u8_kernel(const uint8_t* __restrict__ x, uint64_t n,
                                                                    unsigned long long* __restrict__ hist) {
    __shared__ uint32_t sh[kHistThreads / 32][256];
    uint32_t* mine = sh[threadIdx.x >> 5];
    for (int i = threadIdx.x; i < (kHistThreads / 32) * 256; i += kHistThreads) (&sh[0][0])[i] = 0;
    __syncthreads();
    const uint64_t nvec = n / 16;
    const uint4* xv = reinterpret_cast<const uint4*>(x);
    const uint64_t stride = uint64_t(gridDim.x) * kHistThreads;
    for (uint64_t v = uint64_t(blockIdx.x) * kHistThreads + threadIdx.x; v < nvec; v += stride) {
        const uint4 q = __ldcs(xv + v);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int k = 0; k < 16; k++) atomicAdd(&mine[(w[k >> 2] >> (8 * (k & 3))) & 0xFFu], 1u);
    }
    for (uint64_t i = nvec * 16 + uint64_t(blockIdx.x) * kHistThreads + threadIdx.x; i < n; i += stride)
        atomicAdd(&mine[x[i]], 1u);
    __syncthreads();
    for (int s = threadIdx.x; s < 256; s += kHistThreads) {
        uint64_t t = 0;
        for (int w = 0; w < kHistThreads / 32; w++) t += sh[w][s];
        if (t) atomicAdd(hist + s, (unsigned long long)t);
    }
}

__global__ void __launch_bounds__(kHistThreads) histogram_kernel(const uint16_t* __restrict__ x, uint64_t n,
                                                                 unsigned long long* __restrict__ hist) {
    __shared__ uint32_t sh[kHistThreads / 32][256];
    uint32_t* mine = sh[threadIdx.x >> 5];
    for (int i = threadIdx.x; i < (kHistThreads / 32) * 256; i += kHistThreads) (&sh[0][0])[i] = 0;
    __syncthreads();
    const uint64_t nvec = n / 8;
    const uint4* xv = reinterpret_cast<const uint4*>(x);
    const uint64_t stride = uint64_t(gridDim.x) * kHistThreads;
    for (uint64_t v = uint64_t(blockIdx.x) * kHistThreads + threadIdx.x; v < nvec; v += stride) {
        const uint4 q = __ldcs(xv + v);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int k = 0; k < 4; k++) {
            atomicAdd(&mine[(w[k] >> 7) & 0xFFu], 1u);
            atomicAdd(&mine[(w[k] >> 23) & 0xFFu], 1u);
        }
    }
    for (uint64_t i = nvec * 8 + uint64_t(blockIdx.x) * kHistThreads + threadIdx.x; i < n; i += stride)
        atomicAdd(&mine[(x[i] >> 7) & 0xFFu], 1u);
    __syncthreads();
    for (int s = threadIdx.x; s < 256; s += kHistThreads) {
        uint64_t t = 0;
        for (int w = 0; w < kHistThreads / 32; w++) t += sh[w][s];
        if (t) atomicAdd(hist + s, (unsigned long long)t);
    }
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
    uint2 e[256];  // x = code left-aligned in 32 bits, y = its length (0 = absent)
};

__device__ __forceinline__ void stage_codes(SharedCodes& sc, const CodeTable& ct) {
    for (int v = threadIdx.x; v < 256; v += blockDim.x) {
        const uint32_t l = ct.len[v];
        sc.e[v] = make_uint2(l ? ct.code[v] << (32u - l) : 0u, l);
    }
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
__device__ __forceinline__ RawElems load_raw(const SegTable& sg, uint64_t c0, uint64_t i0, uint64_t n) {
    RawElems r;
    r.direct = false;
    if (i0 < n) {
        uint32_t seg = find_seg(sg, c0);
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

// Bits of code per chunk.
template <int ES>
__global__ void __launch_bounds__(kEncThreads) chunk_bits_kernel(const __grid_constant__ SegTable sg,
                                                                 const __grid_constant__ CodeTable ct,
                                                                 uint64_t n, uint64_t n_chunks,
                                                                 uint32_t* __restrict__ chunk_bits) {
    __shared__ SharedCodes sc;
    __shared__ uint32_t s_warp[kEncThreads / 32];
    stage_codes(sc, ct);
    __syncthreads();
    const uint64_t tofs = uint64_t(threadIdx.x) * kEncPerThread;
    uint64_t c = blockIdx.x;
    RawElems next = load_raw<ES>(sg, c * kEncChunk, c * kEncChunk + tofs, n);
    for (; c < n_chunks; c += gridDim.x) {
        const RawElems cur = next;
        const uint64_t i0 = c * kEncChunk + tofs;
        if (c + gridDim.x < n_chunks)
            next = load_raw<ES>(sg, (c + gridDim.x) * kEncChunk, (c + gridDim.x) * kEncChunk + tofs, n);
        uint32_t bits = 0;
        if (i0 < n) {
            uint32_t w[kWords<ES>];
            raw_words<ES>(sg, cur, i0, n, w);
            const uint64_t left = n - i0;
            bits = thread_bits<ES>(sc, w, left < kEncPerThread ? uint32_t(left) : kEncPerThread);
        }
        uint32_t total;
        block_exclusive_scan<kEncThreads>(bits, s_warp, total);
        if (threadIdx.x == 0) chunk_bits[c] = total;
        __syncthreads();  // s_warp is reused by the next chunk
    }
}

// Exclusive prefix sum of the chunk totals in one CTA, 4096 chunks per tile
// (four per thread, 16-byte loads), the next tile's loads issued before the
// current tile is scanned.
constexpr int kScanThreads = 1024;
__global__ void __launch_bounds__(kScanThreads) chunk_scan_kernel(const uint32_t* __restrict__ chunk_bits,
                                                                  uint64_t n_chunks,
                                                                  unsigned long long* __restrict__ chunk_start) {
    __shared__ unsigned long long s_warp[kScanThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr uint64_t kTile = 4 * kScanThreads;
    auto load4 = [&](uint64_t base) {
        const uint64_t c = base + 4 * uint64_t(threadIdx.x);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (c + 4 <= n_chunks) {
            v = __ldg(reinterpret_cast<const uint4*>(chunk_bits + c));
        } else {
            if (c < n_chunks) v.x = chunk_bits[c];
            if (c + 1 < n_chunks) v.y = chunk_bits[c + 1];
            if (c + 2 < n_chunks) v.z = chunk_bits[c + 2];
            if (c + 3 < n_chunks) v.w = chunk_bits[c + 3];
        }
        return v;
    };
    unsigned long long carry = 0;
    uint4 v = load4(0);
    for (uint64_t base = 0; base < n_chunks; base += kTile) {
        const uint4 cur = v;
        if (base + kTile < n_chunks) v = load4(base + kTile);
        const unsigned long long own = (unsigned long long)cur.x + cur.y + cur.z + cur.w;
        unsigned long long incl = own;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += y;
        }
        if (lane == 31) s_warp[warp] = incl;
        __syncthreads();
        unsigned long long before = 0, total = 0;
        for (int w = 0; w < kScanThreads / 32; w++) {
            const unsigned long long t = s_warp[w];
            total += t;
            before += w < warp ? t : 0ull;
        }
        __syncthreads();  // s_warp is rewritten by the next tile
        unsigned long long run = carry + before + incl - own;
        const uint64_t c = base + 4 * uint64_t(threadIdx.x);
        const uint32_t e[4] = {cur.x, cur.y, cur.z, cur.w};
#pragma unroll
        for (int k = 0; k < 4; k++) {
            if (c + k < n_chunks) chunk_start[c + k] = run;
            run += e[k];
        }
        carry += total;
    }
}

// ---------------------------------------------------------------------------
// Bit-pack.  Each thread appends its codes to a register word with funnel
// shifts; its first word (which it may share with the previous thread) and
// its last, partial word (shared with the next) are OR-ed into a
// shared-memory image of the chunk, the words in between are stored.  The
// image's interior words are then stored to EncodedExponent and its two
// boundary words, shared with the neighbouring chunks, are OR-ed into global
// memory.  The same pass writes the sign+mantissa bytes, each window's gap
// and each thread block's output position from the element's own start bit
// s and length l:
//   * a code that starts inside window w-1 and runs into window w sets
//     gap[w] = s + l - 64w (gaps of windows that begin exactly at a code start
//     stay 0);
//   * a code that starts exactly at bit 64*T*b sets off[b] = i, one that runs
//     over that bit sets off[b] = i + 1.
// Positions are kept 32-bit relative to the chunk's first bit rounded down to
// a thread-block boundary; a code covers a window boundary exactly when
// (u >> 6) changes across it, u = relative start + 63, which is one test per
// element.
// ---------------------------------------------------------------------------
constexpr int kPackWords = kEncChunk + 4;  // 32 bits per element at most, plus the misalignment
// windows a thread's codes can reach into: 16 codes of at most 32 bits
constexpr int kMaxEvents = (int(kEncPerThread) * 32) / 64 + 1;
static_assert(kPackWords % 4 == 0, "image cleared in 16-byte stores");

template <int ES>
__global__ void __launch_bounds__(kEncThreads) pack_kernel(const __grid_constant__ SegTable sg,
                                                           const __grid_constant__ CodeTable ct, uint64_t n,
                                                           uint64_t n_chunks, uint32_t log2_block_bits,
                                                           const unsigned long long* __restrict__ chunk_start,
                                                           uint32_t* __restrict__ exp32, uint8_t* __restrict__ sm,
                                                           uint32_t* __restrict__ gaps32,
                                                           uint32_t* __restrict__ block_off, uint64_t n_blocks,
                                                           uint32_t* __restrict__ chunk_bit) {
    __shared__ SharedCodes sc;
    __shared__ __align__(16) uint32_t s_words[kPackWords];
    __shared__ uint32_t s_ev[kMaxEvents][kEncThreads];
    __shared__ uint32_t s_warp[kEncThreads / 32];
    stage_codes(sc, ct);
    __syncthreads();
    const uint64_t block_mask = (uint64_t(1) << log2_block_bits) - 1;
    const uint64_t tofs = uint64_t(threadIdx.x) * kEncPerThread;
    uint64_t c = blockIdx.x;
    RawElems next = load_raw<ES>(sg, c * kEncChunk, c * kEncChunk + tofs, n);
    for (; c < n_chunks; c += gridDim.x) {
        const RawElems cur = next;
        const uint64_t i0 = c * kEncChunk + tofs;
        if (c + gridDim.x < n_chunks)
            next = load_raw<ES>(sg, (c + gridDim.x) * kEncChunk, (c + gridDim.x) * kEncChunk + tofs, n);
        uint32_t w8[kWords<ES>];
        uint32_t valid = 0, bits = 0;
        if (i0 < n) {
            raw_words<ES>(sg, cur, i0, n, w8);
            const uint64_t left = n - i0;
            valid = left < kEncPerThread ? uint32_t(left) : kEncPerThread;
            bits = thread_bits<ES>(sc, w8, valid);
        }
        for (int j = threadIdx.x; j < kPackWords / 4; j += kEncThreads)
            reinterpret_cast<uint4*>(s_words)[j] = make_uint4(0, 0, 0, 0);
        uint32_t chunk_total;
        const uint32_t my_off = block_exclusive_scan<kEncThreads>(bits, s_warp, chunk_total);
        const uint64_t S = chunk_start[c];
        const uint32_t lead = uint32_t(S & 31u);
        const uint64_t Sb = S & ~block_mask;  // a thread-block (and window) boundary
        // gap and output position for a code at relative start r (bits from
        // Sb) of length l, element i, that covers a window boundary
        const uint64_t gap_base = 5 * (Sb >> 6);
        const uint64_t blk_base = Sb >> log2_block_bits;
        auto window_event = [&](uint32_t r, uint32_t l, uint64_t i) {
            if (r & 63u) {
                const uint32_t wr = (r >> 6) + 1;
                const uint32_t g = r + l - 64 * wr;
                const uint64_t gb = gap_base + 5 * uint64_t(wr);
                const uint32_t sh = uint32_t(gb & 31);
                atomicOr(gaps32 + (gb >> 5), g << sh);
                if (sh > 27) atomicOr(gaps32 + (gb >> 5) + 1, g >> (32 - sh));
            }
            const uint32_t br = r >> log2_block_bits;
            if ((r & uint32_t(block_mask)) == 0) {
                block_off[blk_base + br] = uint32_t(i);
            } else if (((r + l - 1) >> log2_block_bits) != br) {
                block_off[blk_base + br + 1] = uint32_t(i + 1);
            }
        };
        // Append this thread's codes to the image.  A completed word is OR-ed
        // in (the first may be shared with the previous thread).  Codes that
        // cover a window boundary (at most 9 for 16 codes of <= 32 bits) are
        // only noted in the thread's column of s_ev and handled after the
        // loop, so the warp does not run that handler on every element.
        auto pack_codes = [&](auto full_tag) {
            constexpr bool kFull = decltype(full_tag)::value;  // all kEncPerThread elements valid
            const uint32_t q = lead + my_off;  // bit position in the chunk image
            uint32_t w = q >> 5, fill = q & 31u, cur_word = 0;
            uint32_t u = uint32_t(S - Sb) + my_off + 63u;  // relative start + 63
            uint32_t ne = 0;
#pragma unroll
            for (int k = 0; k < int(kEncPerThread); k++) {
                if (!kFull && uint32_t(k) >= valid) break;
                const uint2 ce = sc.e[symbol<ES>(w8, k)];
                const uint32_t t = ce.x, l = ce.y;
                cur_word |= t >> fill;
                const uint32_t spill = __funnelshift_r(0u, t, fill);  // bits that did not fit
                fill += l;
                if (fill >= 32u) {
                    atomicOr(&s_words[w], cur_word);
                    w++;
                    cur_word = spill;
                    fill -= 32u;
                }
                const uint32_t nu = u + l;
                if ((u ^ nu) >= 64u) s_ev[ne++][threadIdx.x] = (u << 10) | (l << 4) | uint32_t(k);
                u = nu;
            }
            if (fill) atomicOr(&s_words[w], cur_word);
            if (gaps32) {
                for (uint32_t j = 0; j < ne; j++) {
                    const uint32_t e = s_ev[j][threadIdx.x];
                    window_event((e >> 10) - 63u, (e >> 4) & 63u, i0 + (e & 15u));
                }
            }
        };
        if (valid == kEncPerThread)
            pack_codes(std::true_type{});
        else if (valid)
            pack_codes(std::false_type{});
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
        __syncthreads();
        const uint32_t nwords = (lead + chunk_total + 31) >> 5;
        const uint64_t W0 = S >> 5;
        for (uint32_t j = threadIdx.x; j < nwords; j += kEncThreads) {
            const uint32_t v = __byte_perm(s_words[j], 0, 0x0123);  // MSB-first bytes
            if (j == 0 || j == nwords - 1) {
                if (v) atomicOr(exp32 + W0 + j, v);
            } else {
                exp32[W0 + j] = v;
            }
        }
        __syncthreads();  // s_words and s_warp are reused by the next chunk
    }
}

// Persistent grid for an encode kernel: as many CTAs as can be resident on
// every SM at once.
template <typename Kernel>
unsigned encode_grid(Kernel kernel, uint64_t chunks) {
    int dev = 0, sms = 148, per_sm = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kEncThreads, 0) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    const uint64_t want = uint64_t(sms) * uint64_t(per_sm);
    return unsigned(chunks < want ? chunks : want);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Workspace {
    unsigned long long* hist;
    uint32_t* chunk_bits;
    unsigned long long* chunk_start;
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
    w->chunk_bits = reinterpret_cast<uint32_t*>(p + 2048);
    w->chunk_start = reinterpret_cast<unsigned long long*>(p + 2048 + align16(4 * chunks));
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

// Histogram kernels (one launch per segment), host code builder, header.
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
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    for (uint32_t k = 0; k < n_segs; k++) {
        const uint64_t cnt = seg_counts[k];
        if (!cnt) continue;
        const uint64_t vec_blocks = (cnt / (16 / ES) + kHistThreads - 1) / kHistThreads;
        uint64_t grid = vec_blocks < uint64_t(4 * sms) ? vec_blocks : uint64_t(4 * sms);
        if (grid == 0) grid = 1;
        if constexpr (ES == 2)
            histogram_kernel<<<unsigned(grid), kHistThreads, 0, s>>>(
                reinterpret_cast<const uint16_t*>(sg.ptr[k]), cnt, w.hist);
        else
            histogram_u8_kernel<<<unsigned(grid), kHistThreads, 0, s>>>(sg.ptr[k], cnt, w.hist);
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
    return df11_header_init(hdr, len, n, bits, threads_per_block, max_code_len, seg_counts, n_segs);
}

// Table upload, clears, then the chunk-bits, scan and bit-pack kernels.
// d_sm is written for BF16 input (ES = 2) only.
// With d_chunk_bit (the independent-chunk table instead of Gaps and block
// offsets) d_gaps and d_block_off are not written and may be null.
template <int ES>
df11_status compress_encode(const char* fn, const void* const* d_segs, const df11_header* hdr,
                            uint32_t* chunk_bits, unsigned long long* chunk_start, uint8_t* d_exp, uint8_t* d_sm,
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
    // decode tables are built in this thread's own host buffer (no heap)
    static thread_local unsigned char lut[kLutBytes];
    st = df11_build_lut(hdr, lut, sizeof(lut));
    if (st != DF11_OK) return st;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if ((e = cudaMemcpyAsync(d_lut, lut, kLutBytes, cudaMemcpyHostToDevice, s)) != cudaSuccess)
        return cuda_fail("table upload", e);
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
    if (n == 0) return DF11_OK;

    const uint64_t chunks = (n + kEncChunk - 1) / kEncChunk;
    if (chunks >= (uint64_t(1) << 31)) return fail(DF11_ERR_TOO_LARGE, "too many chunks");
    chunk_bits_kernel<ES><<<encode_grid(chunk_bits_kernel<ES>, chunks), kEncThreads, 0, s>>>(sg, ct, n, chunks,
                                                                                          chunk_bits);
    chunk_scan_kernel<<<1, kScanThreads, 0, s>>>(chunk_bits, chunks, chunk_start);
    uint32_t log2_bb = 6;
    while ((1u << (log2_bb - 6)) < hdr->threads_per_block) log2_bb++;
    pack_kernel<ES><<<encode_grid(pack_kernel<ES>, chunks), kEncThreads, 0, s>>>(
        sg, ct, n, chunks, log2_bb, chunk_start, reinterpret_cast<uint32_t*>(d_exp), d_sm,
        reinterpret_cast<uint32_t*>(d_gaps), d_block_off, hdr->n_blocks, d_chunk_bit);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("encode launch", e);
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
    return compress_encode<2>("df11_compress_encode", d_segs, hdr, w.chunk_bits, w.chunk_start, d_exp, d_sm, d_gaps,
                              d_block_off, d_lut, stream);
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
    return compress_encode<1>("df11_compress_encode_u8", d_segs, hdr, w.chunk_bits, w.chunk_start, d_exp,
                              nullptr, d_gaps, d_block_off, d_lut, stream);
}

// ---------------------------------------------------------------------------
// Encode without any allocation: the same kernels as df11_compress_encode,
// with their scratch (per-chunk bit totals and chunk start bits) in a
// fixed-size array that lives in the library's own device memory.  For
// callers that cannot allocate device memory when they compress: serving
// engines that hand all of HBM to their own pools at start-up and forbid
// later cudaMalloc calls, and code running inside an allocator (an
// out-of-memory handler, say) where allocating would recurse.
// ---------------------------------------------------------------------------
namespace df11 {
namespace {

constexpr uint64_t kStaticChunks = DF11_STATIC_MAX_ELEMS / kEncChunk;
constexpr uint64_t kStaticBitsBytes = 4 * kStaticChunks;
constexpr uint64_t kStaticScratchBytes = kStaticBitsBytes + 8 * kStaticChunks;
static_assert(DF11_STATIC_MAX_ELEMS % kEncChunk == 0, "whole chunks");

// Loaded with the library on every GPU that uses it and held until exit.
// Every call overwrites all of the scratch it reads, so nothing has to be
// cleared between calls; two calls that overlap on the GPU share it and race.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of the scratch, looked up once per device with that device
// current (host code cannot use the symbol itself as a device pointer).
constexpr int kMaxDevices = 64;
std::atomic<void*> g_static_scratch_addr[kMaxDevices];
std::mutex g_static_scratch_mu;

df11_status static_scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    if (dev < 0 || dev >= kMaxDevices) return fail(DF11_ERR_INVALID, "device ordinal %d above %d", dev, kMaxDevices);
    void* p = g_static_scratch_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_static_scratch_mu);
        p = g_static_scratch_addr[dev].load(std::memory_order_relaxed);
        if (!p) {
            e = cudaGetSymbolAddress(&p, g_static_scratch);
            if (e != cudaSuccess) return cuda_fail("cudaGetSymbolAddress(static scratch)", e);
            g_static_scratch_addr[dev].store(p, std::memory_order_release);
        }
    }
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
    uint32_t* chunk_bits = static_cast<uint32_t*>(scratch);
    unsigned long long* chunk_start =
        reinterpret_cast<unsigned long long*>(static_cast<unsigned char*>(scratch) + kStaticBitsBytes);
    return compress_encode<2>("df11_compress_encode_static", d_segs, hdr, chunk_bits, chunk_start, d_exp, d_sm,
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
    return compress_encode<2>("df11_compress_encode_chunked", d_segs, hdr, w.chunk_bits, w.chunk_start, d_exp,
                              d_sm, nullptr, nullptr, d_lut, stream, d_chunk_bit);
}
