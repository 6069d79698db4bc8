// DF11 decompression kernel for sm_100a.
//
// Follows the two-phase design of "DFloat11: compressao sem perda para
// inferencia em GPU que reduz LLMs para 70% do tamanho", section "Kernel de
// GPU em 2 etapas e metadados auxiliares": every thread owns one 8-byte
// window of EncodedExponent and decodes the codes that start in it, beginning
// at its 5-bit gap; phase 1 counts them, a block-wide prefix sum turns counts
// into output positions (added to the thread block's stored position), and
// phase 2 decodes again into an on-chip buffer that is written to HBM with
// coalesced stores.  One launch covers a whole stream, i.e. every matrix of a
// transformer block ("Descompressao por bloco de transformer").
//
// B200 specifics:
//   * persistent grid (resident CTAs x SMs): the decode tables are copied to
//     shared memory once per CTA and reused for every thread block of the
//     stream;
//   * multi-symbol level-1 tables: the count table gives the start mask of
//     every complete code in the next 12 bits, the decode table up to three
//     symbols per lookup; codes longer than 12 bits use the canonical
//     comparison ladder (level 2);
//   * the merge of exponent and sign+mantissa works on 16 elements per
//     thread: one 16-byte shared load, one 16-byte streaming global load, two
//     16-byte streaming global stores.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdio>

#include "df11_internal.h"

namespace df11 {
namespace {

struct DecodeArgs {
    const uint8_t* exp;
    const uint4* sm;
    const uint32_t* gaps;
    const uint32_t* off;
    const uint4* lut;
    uint16_t* out;
    uint32_t* status;
    uint64_t n_elems;
    uint64_t total_bits;
    uint64_t n_threads;
    uint64_t n_blocks;
};

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

// 32 stream bits starting at bit `pos` (0 <= pos < 64) of the 96-bit window
// w0:w1:w2 (MSB first).
__device__ __forceinline__ uint32_t peek32(uint32_t w0, uint32_t w1, uint32_t w2, int pos) {
    const uint32_t hi = pos < 32 ? w0 : w1;
    const uint32_t lo = pos < 32 ? w1 : w2;
    return __funnelshift_l(lo, hi, uint32_t(pos));
}

// Length of the canonical code at the top of `peek` (level 2); 0 if no code
// matches (only possible in a corrupt stream).
__device__ __forceinline__ int code_length(const unsigned long long* lj_end, uint32_t peek) {
    for (int l = 1; l <= 32; l++)
        if ((unsigned long long)peek < lj_end[l]) return l;
    return 0;
}

// Two BF16 results from exponent bytes and sign+mantissa bytes picked by
// `sel` (0x4140: bytes 0 and 1, 0x4342: bytes 2 and 3):
// bf16 = (sm & 0x80) << 8 | e << 7 | (sm & 0x7F).
__device__ __forceinline__ uint32_t merge_pair(uint32_t e4, uint32_t s4, uint32_t sel) {
    const uint32_t x = __byte_perm(s4, 0, sel);
    const uint32_t e = __byte_perm(e4, 0, sel);
    return (x & 0x007F007Fu) | ((x & 0x00800080u) << 8) | (e << 7);
}

template <int T>
__global__ void __launch_bounds__(T) decode_kernel(const DecodeArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t* s_lut = smem;
    uint8_t* s_stage = smem + kLutBytes;                                    // 64*T + 64 bytes
    uint32_t* s_warp = reinterpret_cast<uint32_t*>(s_stage + 64 * T + 64);  // T/32 words

    for (int i = threadIdx.x; i < int(kLutBytes / 16); i += T)
        reinterpret_cast<uint4*>(s_lut)[i] = a.lut[i];
    __syncthreads();
    const uint16_t* ctab = reinterpret_cast<const uint16_t*>(s_lut + kLutOffCount);
    const uint32_t* dtab = reinterpret_cast<const uint32_t*>(s_lut + kLutOffDecode);
    const unsigned long long* lj_end = reinterpret_cast<const unsigned long long*>(s_lut + kLutOffLjEnd);
    const uint32_t* delta = reinterpret_cast<const uint32_t*>(s_lut + kLutOffDelta);
    const uint8_t* syms = s_lut + kLutOffSyms;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;

    for (uint64_t b = blockIdx.x; b < a.n_blocks; b += gridDim.x) {
        const uint64_t tg = b * T + threadIdx.x;
        uint32_t w0 = 0, w1 = 0, w2 = 0;
        int start = 0, wend = 0;
        if (tg < a.n_threads) {
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(a.exp) + tg);
            const uint32_t v2 = __ldg(reinterpret_cast<const uint32_t*>(a.exp) + 2 * tg + 2);
            w0 = bswap32(v.x);
            w1 = bswap32(v.y);
            w2 = bswap32(v2);
            const uint64_t gbit = 5 * tg;
            const uint32_t glo = __ldg(a.gaps + (gbit >> 5));
            const uint32_t ghi = __ldg(a.gaps + (gbit >> 5) + 1);
            start = int(__funnelshift_r(glo, ghi, uint32_t(gbit)) & 31u);
            const uint64_t rem = a.total_bits - 64 * tg;
            wend = rem < 64 ? int(rem) : 64;
        }
        const uint32_t off_b = __ldg(a.off + b);
        const uint32_t off_b1 = __ldg(a.off + b + 1);

        // ---- phase 1: count the codes that start in the window ----------
        uint32_t cnt = 0;
        bool bad = false;
        for (int p = start; p < wend;) {
            const uint32_t pk = peek32(w0, w1, w2, p);
            const uint32_t e = ctab[pk >> (32 - kCountBits)];
            if (e) {
                uint32_t m = e & 0xFFFu;
                const int lim = wend - p;
                if (lim < kCountBits) m &= (1u << lim) - 1u;
                cnt += __popc(m);
                p += int(e >> 12);
            } else {
                const int l = code_length(lj_end, pk);
                if (!l) {
                    bad = true;
                    break;
                }
                cnt += 1;
                p += l;
            }
        }

        // ---- block-wide exclusive scan of the counts --------------------
        uint32_t incl = cnt;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += y;
        }
        if (lane == 31) s_warp[warp] = incl;
        const int any_bad = __syncthreads_or(bad);
        uint32_t before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < T / 32; w++) {
            const uint32_t v = s_warp[w];
            total += v;
            before += (w < warp) ? v : 0u;
        }
        const uint32_t excl = before + incl - cnt;
        if (any_bad || off_b1 < off_b || total != off_b1 - off_b || uint64_t(off_b1) > a.n_elems) {
            if (threadIdx.x == 0 && a.status) atomicOr(a.status, uint32_t(DF11_ERR_CORRUPT));
            __syncthreads();
            continue;
        }

        // ---- phase 2: decode again into the staging buffer ---------------
        // staging byte 0 holds element off_b rounded down to 16
        const uint32_t head = off_b & 15u;
        uint8_t* st = s_stage + head + excl;
        {
            int p = start;
            for (uint32_t w = 0; w < cnt;) {
                const uint32_t pk = peek32(w0, w1, w2, p);
                const uint32_t e = dtab[pk >> (32 - kDecodeBits)];
                uint32_t n = (e >> 24) & 3u;
                uint32_t s3 = e;
                if (n) {
                    p += int(e >> 26);
                } else {
                    int l = code_length(lj_end, pk);
                    l = l ? l : 1;
                    s3 = syms[((pk >> (32 - l)) + delta[l]) & 0xFFu];
                    n = 1;
                    p += l;
                }
                const uint32_t r = cnt - w;
                n = n < r ? n : r;
                st[w] = uint8_t(s3);
                if (n > 1) st[w + 1] = uint8_t(s3 >> 8);
                if (n > 2) st[w + 2] = uint8_t(s3 >> 16);
                w += n;
            }
        }
        __syncthreads();

        // ---- merge with sign+mantissa, 16 elements per thread ------------
        const uint64_t c0 = off_b >> 4;
        const uint64_t c1 = (uint64_t(off_b1) + 15) >> 4;
        for (uint64_t c = c0 + threadIdx.x; c < c1; c += T) {
            const uint4 ev = *reinterpret_cast<const uint4*>(s_stage + 16 * (c - c0));
            const uint4 sv = __ldcs(a.sm + c);
            uint4 o0, o1;
            o0.x = merge_pair(ev.x, sv.x, 0x4140);
            o0.y = merge_pair(ev.x, sv.x, 0x4342);
            o0.z = merge_pair(ev.y, sv.y, 0x4140);
            o0.w = merge_pair(ev.y, sv.y, 0x4342);
            o1.x = merge_pair(ev.z, sv.z, 0x4140);
            o1.y = merge_pair(ev.z, sv.z, 0x4342);
            o1.z = merge_pair(ev.w, sv.w, 0x4140);
            o1.w = merge_pair(ev.w, sv.w, 0x4342);
            const uint64_t i0 = 16 * c;
            uint16_t* dst = a.out + i0;
            if (i0 >= off_b && i0 + 16 <= off_b1) {
                __stcs(reinterpret_cast<uint4*>(dst), o0);
                __stcs(reinterpret_cast<uint4*>(dst) + 1, o1);
            } else {
                const uint32_t words[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
#pragma unroll
                for (int k = 0; k < 16; k++) {
                    const uint64_t i = i0 + k;
                    if (i >= off_b && i < off_b1) dst[k] = uint16_t(words[k >> 1] >> (16 * (k & 1)));
                }
            }
        }
        __syncthreads();
    }
}

template <int T>
constexpr size_t decode_smem_bytes() {
    return kLutBytes + 64 * T + 64 + 4 * (T / 32);
}

struct LaunchInfo {
    std::atomic<int> ready{0};
    int grid_per_sm = 0;
    int sms = 0;
};
LaunchInfo g_info[16][5];  // [device][log2(T) - 6]

template <int T>
df11_status launch_decode(const DecodeArgs& a, cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16)
        return fail(DF11_ERR_CUDA, "cudaGetDevice failed");
    constexpr int slot = (T == 64) ? 0 : (T == 128) ? 1 : (T == 256) ? 2 : (T == 512) ? 3 : 4;
    LaunchInfo& li = g_info[dev][slot];
    const size_t smem = decode_smem_bytes<T>();
    if (!li.ready.load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(smem));
        if (e != cudaSuccess) return fail(DF11_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        int per_sm = 0, sms = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<T>, T, smem);
        if (e != cudaSuccess) return fail(DF11_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(e));
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return fail(DF11_ERR_CUDA, "SM count: %s", cudaGetErrorString(e));
        li.grid_per_sm = per_sm > 0 ? per_sm : 1;
        li.sms = sms;
        li.ready.store(1, std::memory_order_release);
    }
    const uint64_t want = uint64_t(li.grid_per_sm) * uint64_t(li.sms);
    const unsigned grid = unsigned(a.n_blocks < want ? a.n_blocks : want);
    decode_kernel<T><<<grid, T, smem, stream>>>(a);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(DF11_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
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
    if (T < 64 || T > 1024 || (T & (T - 1))) return fail(DF11_ERR_INVALID, "threads_per_block %u", T);
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

extern "C" df11_status df11_decompress(const df11_header* hdr, const uint8_t* d_exp, const uint8_t* d_sm,
                                       const uint8_t* d_gaps, const uint32_t* d_block_off,
                                       const void* d_lut, uint16_t* d_out, uint32_t* d_status,
                                       void* stream) {
    df11_status st = check_header(hdr);
    if (st != DF11_OK) return st;
    if (hdr->n_elems == 0) return DF11_OK;
    if (!d_exp || !d_sm || !d_gaps || !d_block_off || !d_lut || !d_out)
        return fail(DF11_ERR_INVALID, "df11_decompress: null device pointer");
    if (!aligned16(d_exp) || !aligned16(d_sm) || !aligned16(d_gaps) || !aligned16(d_block_off) ||
        !aligned16(d_lut) || !aligned16(d_out))
        return fail(DF11_ERR_INVALID, "df11_decompress: device pointers must be 16-byte aligned");
    DecodeArgs a;
    a.exp = d_exp;
    a.sm = reinterpret_cast<const uint4*>(d_sm);
    a.gaps = reinterpret_cast<const uint32_t*>(d_gaps);
    a.off = d_block_off;
    a.lut = reinterpret_cast<const uint4*>(d_lut);
    a.out = d_out;
    a.status = d_status;
    a.n_elems = hdr->n_elems;
    a.total_bits = hdr->total_bits;
    a.n_threads = hdr->n_threads;
    a.n_blocks = hdr->n_blocks;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (hdr->threads_per_block) {
        case 64: return launch_decode<64>(a, s);
        case 128: return launch_decode<128>(a, s);
        case 256: return launch_decode<256>(a, s);
        case 512: return launch_decode<512>(a, s);
        case 1024: return launch_decode<1024>(a, s);
        default: return fail(DF11_ERR_INVALID, "threads_per_block %u", hdr->threads_per_block);
    }
}
