/*
 * df11.h -- C ABI of the DF11 (DFloat11) codec for BF16 weights on B200.
 *
 * What the format is ("DFloat11: compressao sem perda para inferencia em GPU
 * que reduz LLMs para 70% do tamanho", section "O formato DFloat11"; abstract
 * of "70% Size, 100% Accuracy: Lossless LLM Compression for Efficient GPU
 * Inference via Dynamic-Length Float"): every BF16 value is split into its
 * 8-bit exponent and a byte holding sign and mantissa.  The exponents are
 * Huffman-coded into the bit-packed EncodedExponent array; the sign+mantissa
 * bytes are kept raw in PackedSignMantissa.  Decoding rebuilds the original
 * BF16 bits exactly.
 *
 * Decoder metadata (section "Kernel de GPU em 2 etapas e metadados
 * auxiliares"): each GPU thread owns an 8-byte window of EncodedExponent and
 * decodes the codes that start in it; a 5-bit Gaps entry per thread gives the
 * offset of its first code, and one 32-bit output position per thread block
 * gives where the block's decoded elements go.
 *
 * Byte layout (readings of points the pages leave open):
 *   - PackedSignMantissa byte = sign << 7 | mantissa (7 bits).
 *   - EncodedExponent is MSB-first: stream bit p is bit 7 - p%8 of byte p/8.
 *   - Codes are canonical: present exponents sorted by (length, value), the
 *     first code is all zeros, each next code is (previous + 1) shifted left
 *     by the length increase.  Lengths are the optimal prefix code with at
 *     most max_code_len (<= 32) bits, computed by package-merge; on equal
 *     counts the lower exponent value counts as the lighter symbol, and a
 *     leaf sorts before a package of equal weight.  One present exponent
 *     gets the 1-bit code "0".
 *   - n_threads = ceil(total_bits / 64), n_blocks = ceil(n_threads / T).
 *   - Gaps: n_threads 5-bit fields, field t at array bits 5t..5t+4, array bit
 *     q being bit q%8 of byte q/8.  gap[t] = (first code start >= 64t, or
 *     total_bits if none) - 64t, always in [0, 31].
 *   - Block offsets: uint32 off[n_blocks + 1]; off[b] = number of codes that
 *     start before stream bit 64*T*b; off[n_blocks] = n_elems.
 *   - Buffer sizes (all zero-padded): bytes_exp = 8*T*n_blocks + 16,
 *     bytes_sm = n_elems rounded up to 16, bytes_gaps = ceil(5*T*n_blocks/8)
 *     + 8 rounded up to 16, bytes_off = 4*(n_blocks + 1).
 *
 * Ownership: every buffer belongs to the caller.  Device pointers must be
 * 16-byte aligned.  No entry point allocates device memory; the compress
 * entry points use a caller-provided device workspace.
 *
 * Errors: every call returns a df11_status; nothing aborts or throws across
 * the ABI.  df11_last_error() returns a message for the last failing call on
 * the calling host thread.  A stream that is inconsistent with its metadata is
 * reported by the kernel through the optional device status word (a bitwise
 * OR of df11_status values, 0 when clean) and never traps.
 */
#ifndef DF11_H
#define DF11_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DF11_VERSION 1
#define DF11_WINDOW_BYTES 8
#define DF11_MAX_CODE_LEN 32
#define DF11_MAX_SEGMENTS 64
#define DF11_STATIC_MAX_ELEMS (1ull << 28) /* limit of df11_compress_encode_static */

typedef enum {
    DF11_OK = 0,
    DF11_ERR_INVALID = 1,   /* bad argument, misaligned pointer, bad table   */
    DF11_ERR_CUDA = 2,      /* a CUDA runtime call failed                    */
    DF11_ERR_CORRUPT = 3,   /* stream disagrees with its Gaps / block offsets */
    DF11_ERR_TOO_LARGE = 4, /* n_elems >= 2^32 (block offsets are 32-bit)    */
    DF11_ERR_CAPACITY = 5   /* a buffer is smaller than the header needs     */
} df11_status;

/* Host-side description of one DF11 stream: one matrix, or every matrix of a
 * transformer block concatenated in order (one shared code table). */
typedef struct {
    uint32_t version;            /* DF11_VERSION                               */
    uint32_t window_bytes;       /* 8                                          */
    uint32_t threads_per_block;  /* T: 32, 64, ..., 1024 (library default 64) */
    uint32_t max_code_len;       /* L used to build the code, 1..32            */
    uint64_t n_elems;            /* BF16 elements, < 2^32                      */
    uint64_t total_bits;         /* bits in EncodedExponent                    */
    uint64_t n_threads;          /* ceil(total_bits / 64)                      */
    uint64_t n_blocks;           /* ceil(n_threads / T)                        */
    uint8_t code_len[256];       /* code length per exponent value, 0 = absent */
    uint32_t n_segments;         /* matrices in the stream, 1..64              */
    uint32_t plan_token;         /* set by df11_compress_plan (0 otherwise):
                                    names the per-range histograms it left in
                                    its workspace; df11_compress_encode with
                                    that workspace uses them instead of
                                    counting code bits in a pass of its own    */
    uint64_t seg_elem_off[DF11_MAX_SEGMENTS + 1]; /* segment k = elements
                                    [seg_elem_off[k], seg_elem_off[k+1])       */
    uint64_t bytes_exp;          /* EncodedExponent buffer size                */
    uint64_t bytes_sm;           /* PackedSignMantissa buffer size             */
    uint64_t bytes_gaps;         /* Gaps buffer size                           */
    uint64_t bytes_off;          /* block offsets buffer size                  */
    uint64_t bytes_lut;          /* decode tables size (df11_build_lut)        */
} df11_header;

/* Library version (DF11_VERSION). */
int df11_version(void);

/* Message for the last failing call on this host thread ("" if none). */
const char* df11_last_error(void);

/* Optimal length-limited code lengths for an exponent histogram
 * ("O formato DFloat11": a Huffman code over the exponent distribution, here
 * with at most max_code_len bits).  Host only, no GPU needed.
 *   hist[256]      in: count per exponent value
 *   max_code_len   in: 1..32, 2^max_code_len >= number of present values
 *   code_len[256]  out: length per value, 0 where hist is 0
 * Returns DF11_ERR_INVALID on a bad limit. */
df11_status df11_code_lengths(const uint64_t* hist, uint32_t max_code_len, uint8_t* code_len);

/* Fill a header for a given code table and sizes (used for streams made
 * elsewhere, e.g. read from disk).  Host only.
 *   code_len[256]       in: lengths; must form a prefix code (Kraft <= 1,
 *                           equality required for >= 2 present values)
 *   n_elems, total_bits in: element count (< 2^32) and stream length in bits
 *   threads_per_block   in: T (32..1024, power of two)
 *   seg_counts[n_segs]  in: elements per segment, summing to n_elems; NULL
 *                           with n_segs = 1 means one segment
 * Validates and fills every size field, including bytes_lut. */
df11_status df11_header_init(df11_header* hdr, const uint8_t* code_len, uint64_t n_elems,
                             uint64_t total_bits, uint32_t threads_per_block,
                             uint32_t max_code_len, const uint64_t* seg_counts,
                             uint32_t n_segs);

/* Build the decoder's tables for hdr->code_len into host memory h_lut
 * (capacity cap >= hdr->bytes_lut).  The caller copies them to the device
 * once per stream; df11_decompress reads them from there.  Host only.
 * (Section "Decodificacao com LUT hierarquica": compact lookup tables that
 * fit in on-chip memory, used instead of a bit-level tree walk.) */
df11_status df11_build_lut(const df11_header* hdr, void* h_lut, uint64_t cap);

/* Device workspace the compress entry points need for n_elems elements. */
df11_status df11_compress_workspace_size(uint64_t n_elems, uint64_t* bytes);

/* Compress, step 1 of 2 ("O formato DFloat11"): exponent histogram on the
 * GPU, then the code built on the host; fills *hdr (code_len, total_bits and
 * every buffer size).  Synchronises `stream` once (histogram readback).
 *   d_segs[n_segs]      in: device pointers to BF16 data, 16-byte aligned
 *   seg_counts[n_segs]  in: elements per segment (sum < 2^32); n_segs 1..64
 *   threads_per_block   in: T; max_code_len in: L (1..32; 32 = the pages')
 *   d_workspace         in: device scratch of >= workspace_bytes bytes
 *   stream              in: cudaStream_t (NULL = default stream) */
df11_status df11_compress_plan(const void* const* d_segs, const uint64_t* seg_counts,
                               uint32_t n_segs, uint32_t threads_per_block,
                               uint32_t max_code_len, void* d_workspace,
                               uint64_t workspace_bytes, df11_header* hdr, void* stream);

/* Compress, step 2 of 2: bit-pack kernel.  Writes EncodedExponent,
 * PackedSignMantissa, Gaps and block offsets into caller buffers of at least
 * the header's sizes, and the decode tables into d_lut (hdr->bytes_lut).
 * Asynchronous on `stream`; d_segs must hold the data the plan saw.  With
 * the workspace the plan filled (and its header) the kernel takes each
 * range's code bits from the plan's per-range histograms; any other
 * workspace of the needed size gives the same output, reading the input
 * once more to count them. */
df11_status df11_compress_encode(const void* const* d_segs, const df11_header* hdr,
                                 void* d_workspace, uint64_t workspace_bytes, uint8_t* d_exp,
                                 uint8_t* d_sm, uint8_t* d_gaps, uint32_t* d_block_off,
                                 void* d_lut, void* stream);

/* Compress, step 2 of 2, without allocating: the pages have no counterpart
 * to this entry point.  It writes exactly what df11_compress_encode writes,
 * but keeps its scratch (look-back descriptors, chunk ticket, abort flag) in a fixed
 * array inside the library instead of a caller workspace.  It is for callers
 * that cannot allocate device memory at compress time: serving engines that
 * hand all of HBM to their own pools at start-up and forbid later cudaMalloc
 * calls, and code running inside an allocator (an out-of-memory handler, for
 * instance) where allocating would recurse.  It calls no cudaMalloc/cudaFree.
 *   - At most DF11_STATIC_MAX_ELEMS (2^28) elements per call; larger streams
 *     get DF11_ERR_TOO_LARGE (use df11_compress_encode with a workspace).
 *   - The scratch is 524,304 bytes of device memory that every GPU using the
 *     library's device code holds until exit.
 *   - That device code, and the scratch with it, is put on a GPU when the
 *     library first uses the GPU (CUDA loads modules lazily by default), and
 *     that first use may itself need device memory.  So make one call of this
 *     entry point (or any compress or decompress) on each device at start-up,
 *     before handing HBM to other pools and before any stream capture.
 *   - Every call looks up the scratch's address for the current device and
 *     context on the host; once the device code is loaded this allocates
 *     nothing.
 *   - All calls share the one scratch array, which keeps the last call's
 *     contents; every call clears, on its stream, the part it uses before
 *     its kernel.  Calls whose work overlaps on the GPU (other streams, other
 *     host threads) race on it and must be serialised by the caller.
 * Arguments as for df11_compress_encode, minus the workspace. */
df11_status df11_compress_encode_static(const void* const* d_segs, const df11_header* hdr,
                                        uint8_t* d_exp, uint8_t* d_sm, uint8_t* d_gaps,
                                        uint32_t* d_block_off, void* d_lut, void* stream);

/* Decompress one stream -- every matrix of a transformer block -- in one
 * kernel launch ("Descompressao por bloco de transformer"; two-phase kernel of
 * "Kernel de GPU em 2 etapas e metadados auxiliares").
 *   d_exp, d_sm, d_gaps, d_block_off  in: the stream's device arrays
 *   d_lut       in: device copy of df11_build_lut's output for this header
 *   d_out       out: n_elems BF16 values (uint16 bit patterns), contiguous;
 *               segment k starts at element seg_elem_off[k]
 *   d_status    in/out, may be NULL: device word OR-ed with DF11_ERR_CORRUPT
 *               if the stream disagrees with its metadata (the caller zeroes it)
 *   stream      cudaStream_t (NULL = default stream)
 * Asynchronous: no allocation, no host synchronisation.  n_elems = 0 is a
 * no-op. */
df11_status df11_decompress(const df11_header* hdr, const uint8_t* d_exp, const uint8_t* d_sm,
                            const uint8_t* d_gaps, const uint32_t* d_block_off,
                            const void* d_lut, uint16_t* d_out, uint32_t* d_status,
                            void* stream);

/* df11_decompress on at most max_sms SMs.  The pages decompress a
 * transformer block's matrices as one batch right before that block's
 * forward pass and drop the BF16 copy after the matrix multiplications
 * ("Descompressao adaptada para inferencia em GPU", "Descompressao por bloco
 * de transformer"); decoding block i+1 while block i computes on another
 * CUDA stream is our extension of that pattern, and this entry point lets
 * the decode leave the remaining SMs to the computation (the decode kernel
 * keeps one CTA resident per SM for the whole launch, using all of that SM's
 * registers).  Same arguments, result and asynchrony as df11_decompress;
 * max_sms above the device's SM count means all SMs; max_sms = 0 is
 * DF11_ERR_INVALID. */
df11_status df11_decompress_sms(const df11_header* hdr, const uint8_t* d_exp, const uint8_t* d_sm,
                                const uint8_t* d_gaps, const uint32_t* d_block_off,
                                const void* d_lut, uint16_t* d_out, uint32_t* d_status,
                                uint32_t max_sms, void* stream);

/* Streams of 8-bit symbols coded whole: the codec of "EntroLLM: Compressao
 * de Pesos Codificada por Entropia para Inferencia Eficiente de Modelos de
 * Linguagem Grandes em Dispositivos de Borda" (section "Metodologia", items 2
 * and 3: Huffman coding of the quantized integer weights, decoded in
 * parallel) on this library's container.  The symbol of each element is its
 * whole byte (e.g. a per-tensor quantized weight) and there is no
 * PackedSignMantissa array; EncodedExponent, Gaps, block offsets, the code
 * table, the header and its sizes are as for BF16 streams (bytes_sm is not
 * used).  Arguments as for the BF16 calls, with segments of n bytes.
 * T must be 32 or 64, or 128 when no code is 1 bit long (df11_decompress_u8
 * returns DF11_ERR_INVALID otherwise). */
df11_status df11_compress_plan_u8(const void* const* d_segs, const uint64_t* seg_counts, uint32_t n_segs,
                                  uint32_t threads_per_block, uint32_t max_code_len, void* d_workspace,
                                  uint64_t workspace_bytes, df11_header* hdr, void* stream);
df11_status df11_compress_encode_u8(const void* const* d_segs, const df11_header* hdr, void* d_workspace,
                                    uint64_t workspace_bytes, uint8_t* d_exp, uint8_t* d_gaps,
                                    uint32_t* d_block_off, void* d_lut, void* stream);
/* d_out: n_elems bytes, 16-byte aligned; asynchronous, no allocation. */
df11_status df11_decompress_u8(const df11_header* hdr, const uint8_t* d_exp, const uint8_t* d_gaps,
                               const uint32_t* d_block_off, const void* d_lut, uint8_t* d_out,
                               uint32_t* d_status, void* stream);

/* Decompress thread blocks [block_begin, block_end) of a stream only.  The
 * per-block output positions of "Kernel de GPU em 2 etapas e metadados
 * auxiliares" make every thread block decodable on its own, so a stream can
 * be decoded piece by piece, e.g. while the next piece is still being copied
 * to the device and the previous one copied back (our extension; the pages
 * decode a whole block of matrices at once).  Pointers as for
 * df11_decompress / df11_decompress_u8: the whole stream's arrays, of which
 * the call reads, for b0 = block_begin, b1 = block_end:
 *   d_exp        bytes [8 T b0, 8 T b1 + 16), within bytes_exp
 *   d_gaps       bytes [5 T b0 / 8, 5 T b1 / 8 + 8), within bytes_gaps
 *   d_block_off  entries b0 .. b1
 *   d_sm         bytes [off[b0] rounded down to 128, off[b1] rounded up to 16),
 *                within bytes_sm; only bytes [off[b0], off[b1]) affect d_out
 *   d_lut        all of it
 * and writes exactly output elements [off[b0], off[b1]) of d_out (the whole
 * stream's output buffer); other elements are left as they are, so calls on
 * disjoint ranges may run concurrently into one buffer.  block_begin ==
 * block_end is a no-op; block_begin > block_end or block_end > n_blocks is
 * DF11_ERR_INVALID.  Asynchronous, no allocation. */
df11_status df11_decompress_blocks(const df11_header* hdr, const uint8_t* d_exp, const uint8_t* d_sm,
                                   const uint8_t* d_gaps, const uint32_t* d_block_off, const void* d_lut,
                                   uint16_t* d_out, uint64_t block_begin, uint64_t block_end,
                                   uint32_t* d_status, void* stream);
df11_status df11_decompress_u8_blocks(const df11_header* hdr, const uint8_t* d_exp, const uint8_t* d_gaps,
                                      const uint32_t* d_block_off, const void* d_lut, uint8_t* d_out,
                                      uint64_t block_begin, uint64_t block_end, uint32_t* d_status,
                                      void* stream);

/* Independent chunks: a variant of the container for comparison with the
 * Gaps-and-block-offsets design ("EntroLLM: Compressao de Pesos Codificada
 * por Entropia ...", section "Metodologia", item 3, decodes independently
 * decodable segments in parallel).  Instead of Gaps and block offsets the
 * stream carries chunk_bit[k] = the start bit of element 64 k's code, for
 * k = 0 .. ceil(n/64) - 1, and chunk_bit[ceil(n/64)] = total_bits (uint32;
 * total_bits must be below 2^32).  EncodedExponent, PackedSignMantissa, the
 * header (from df11_compress_plan) and the decode tables are the DF11
 * stream's.  A chunk decodes with no gap, count or prefix sum.
 * df11_compress_encode_chunked writes d_exp, d_sm, d_lut as
 * df11_compress_encode does and d_chunk_bit (4 (ceil(n/64) + 1) bytes,
 * 16-byte aligned); df11_decompress_chunked rebuilds the n BF16 values
 * (d_out, 16-byte aligned), asynchronously, with no allocation. */
df11_status df11_compress_encode_chunked(const void* const* d_segs, const df11_header* hdr, void* d_workspace,
                                         uint64_t workspace_bytes, uint8_t* d_exp, uint8_t* d_sm,
                                         uint32_t* d_chunk_bit, void* d_lut, void* stream);
df11_status df11_decompress_chunked(const df11_header* hdr, const uint8_t* d_exp, const uint8_t* d_sm,
                                    const uint32_t* d_chunk_bit, const void* d_lut, uint16_t* d_out,
                                    uint32_t* d_status, void* stream);

/* Options of df11_decompress_opts (all zero = exactly df11_decompress /
 * df11_decompress_u8).  The pages' first-level tables have 256 entries
 * ("Decodificacao com LUT hierarquica"); the library's default is a 12-bit,
 * multi-symbol table in one shared-memory copy, which measured fastest on
 * LLM weights.  peek_bits selects the alternatives for comparison. */
typedef struct {
    uint32_t peek_bits;          /* 0 or 12: default table; 8, 9 or 10: a 2^K-entry
                                    first-level table held in 16 copies, one per
                                    8-byte bank pair (BF16 streams, T = 64, codes of
                                    >= 2 bits; DF11_ERR_INVALID otherwise)       */
    uint32_t max_sms;            /* 0 = every SM; else size the grid for this many */
    uint32_t max_warps_per_cta;  /* 0 = the kernel's maximum                      */
    uint32_t ctas;               /* 0 = one persistent CTA per SM (fewer for small
                                    streams); else this many CTAs at most, each
                                    decoding a contiguous run of thread blocks --
                                    more CTAs than fit at once simply queue, so
                                    many small CTAs interleave with other kernels */
    uint32_t block_begin;        /* block_begin = block_end = 0: every thread    */
    uint32_t block_end;          /* block; else thread blocks [block_begin,
                                    block_end) only, exactly as
                                    df11_decompress_blocks (same reads, writes
                                    only those blocks' output elements)          */
    uint32_t early_staging;      /* 1: the caller states that the kernel launched
                                    right before this decode on the stream writes
                                    none of this stream's arrays (tables, exponent
                                    stream, gaps, offsets, sign+mantissa bytes) --
                                    the previous block's decode, say, or a consumer
                                    GEMM.  The warp kernel then stages its tables
                                    and first loads while that kernel finishes and
                                    waits for it only before it writes (B200's
                                    programmatic dependent launch).  0 = wait
                                    first (other values: DF11_ERR_INVALID)        */
    uint32_t reserved;           /* must be zero                                  */
} df11_decode_options;

/* df11_decompress (symbols_u8 = 0, d_out: n_elems uint16) or
 * df11_decompress_u8 (symbols_u8 = 1, d_out: n_elems bytes, d_sm unused) with
 * the options above; same arguments otherwise, same result (every option gives
 * bit-identical output), asynchronous, no allocation. */
df11_status df11_decompress_opts(const df11_header* hdr, const uint8_t* d_exp, const uint8_t* d_sm,
                                 const uint8_t* d_gaps, const uint32_t* d_block_off, const void* d_lut,
                                 void* d_out, uint32_t symbols_u8, const df11_decode_options* opt,
                                 uint32_t* d_status, void* stream);

/* Which decode kernel a stream gets on the current device, and its launch
 * shape: a host-side query with no launch and no allocation (the first query
 * for a kernel on a device sets its shared-memory limit and reads its
 * occupancy, as the first decode does).  The pages have no counterpart; it
 * reports the on-chip choices of "Decodificacao com LUT hierarquica" (the
 * width of the first-level table and how many copies of it shared memory
 * holds) and of "Kernel de GPU em 2 etapas e metadados auxiliares" (threads
 * per CTA, CTAs) for a whole-stream df11_decompress / df11_decompress_u8.
 *   hdr         in: the stream's header (checked as df11_decompress checks it)
 *   symbols_u8  in: 0 for BF16 streams, 1 for streams of 8-bit symbols
 *   opt         in, may be NULL: options as for df11_decompress_opts
 *   info        out: see the fields
 * Returns DF11_ERR_INVALID for a header no kernel decodes. */
typedef struct {
    char kernel[64];          /* kernel name with its template arguments        */
    uint32_t grid;            /* CTAs                                            */
    uint32_t block;           /* threads per CTA                                 */
    uint32_t smem_bytes;      /* dynamic shared memory per CTA                   */
    uint32_t peek_bits;       /* first-level table index width K (2^K entries)   */
    uint32_t table_copies;    /* copies of the first-level decode table per CTA  */
    uint32_t reserved;
    uint64_t thread_blocks;   /* format thread blocks (n_blocks)                 */
} df11_kernel_info;
df11_status df11_decode_kernel_info(const df11_header* hdr, uint32_t symbols_u8, const df11_decode_options* opt,
                                    df11_kernel_info* info);

#ifdef __cplusplus
}
#endif

#endif /* DF11_H */
