"""DF11 (DFloat11) lossless BF16 weight codec for NVIDIA B200 (sm_100a).

The codec runs in libdf11.so (hand-written CUDA kernels plus a C++ code
builder behind the C ABI of include/df11.h); this package allocates
caller-owned buffers with PyTorch and passes pointers.  Importing it does not
load the library; the first call does, and raises if it is missing.
"""
from .codec import (DEFAULT_THREADS_PER_BLOCK, IND_CHUNK, ChunkedStream, CompressedStream, HostStream, build_lut,
                    chunked_from_arrays, code_lengths, compress, compress_chunked, compress_u8, decode_options, decompress,
                    decompress_blocks, decompress_chunked, decompress_u8, from_arrays, make_header, piece_ranges,
                    to_host, workspace_bytes)
from ._binding import DF11Error, EXPORTED, load as load_library, library_path
from .prefetch import BlockPrefetcher

__all__ = ["DEFAULT_THREADS_PER_BLOCK", "CompressedStream", "HostStream", "build_lut", "code_lengths", "compress", "decompress",
           "decode_options",
           "compress_u8", "decompress_u8", "IND_CHUNK", "ChunkedStream", "compress_chunked", "decompress_chunked",
           "chunked_from_arrays", "decompress_blocks", "piece_ranges",
           "from_arrays", "make_header", "to_host", "workspace_bytes", "DF11Error", "EXPORTED",
           "load_library", "library_path", "BlockPrefetcher"]
