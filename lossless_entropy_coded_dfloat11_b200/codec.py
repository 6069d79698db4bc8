"""PyTorch-facing API of the DF11 codec.

PyTorch provides device memory and streams; every step of compression and
decompression runs in libdf11.so (CUDA kernels for sm_100a plus the host-side
code builder).  The functions here only allocate caller-owned buffers with
torch and pass raw pointers through the C ABI of include/df11.h.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, field

import numpy as np
import torch

from . import _binding as B

# Thread blocks of one warp: the decode kernel then needs no CTA-wide barrier
# (the block offsets cost 4 bytes per 32 windows, ~0.2% of the stream).
DEFAULT_THREADS_PER_BLOCK = 64


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(int(stream.cuda_stream))


def _ptr(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(int(t.data_ptr()))


def _np_ptr(a: np.ndarray) -> ctypes.c_void_p:
    return ctypes.c_void_p(int(a.ctypes.data))


@dataclass
class CompressedStream:
    """One DF11 stream on the device: a matrix, or every matrix of a
    transformer block sharing one code table."""
    header: B.Header
    exp: torch.Tensor        # uint8  EncodedExponent
    sm: torch.Tensor         # uint8  PackedSignMantissa
    gaps: torch.Tensor       # uint8  5-bit Gaps
    block_off: torch.Tensor  # int32 storage of uint32 block offsets
    lut: torch.Tensor        # uint8  decode tables (df11_build_lut)
    names: list = field(default_factory=list)
    shapes: list = field(default_factory=list)
    symbols: str = "bf16"    # "bf16": BF16 weights; "u8": 8-bit symbols coded whole (no sm array)

    @property
    def n_elems(self) -> int:
        return int(self.header.n_elems)

    @property
    def total_bits(self) -> int:
        return int(self.header.total_bits)

    @property
    def threads_per_block(self) -> int:
        return int(self.header.threads_per_block)

    @property
    def code_len(self) -> np.ndarray:
        return np.frombuffer(bytes(self.header.code_len), dtype=np.uint8).copy()

    def compressed_bytes(self) -> int:
        """Bytes of the format's arrays without padding: code bits, one byte
        per element, 5 bits per thread, 4 bytes per thread-block position and
        the 256-byte code-length table."""
        h = self.header
        side = h.n_elems if self.symbols == "bf16" else 0
        return ((h.total_bits + 7) // 8 + side + (5 * h.n_threads + 7) // 8
                + 4 * (h.n_blocks + 1) + 256)

    def read_bytes(self) -> int:
        """Bytes of the format's arrays one decompress reads (exponent
        stream, sign+mantissa bytes, gaps, block offsets); the decode tables,
        fetched once per CTA and served from L2, are not counted."""
        h = self.header
        side = h.n_elems if self.symbols == "bf16" else 0
        return (h.total_bits + 7) // 8 + side + (5 * h.n_threads + 7) // 8 + 4 * (h.n_blocks + 1)

    def kernel_info(self, u8: bool | None = None, options=None) -> dict:
        """The decode kernel a whole-stream decompress of this stream launches
        on the current device, with its grid, CTA size, shared memory, table
        width and table copies (df11_decode_kernel_info)."""
        info = B.KernelInfo()
        u8 = self.symbols == "u8" if u8 is None else u8
        B.call("df11_decode_kernel_info", ctypes.byref(self.header), 1 if u8 else 0,
               ctypes.byref(options) if options is not None else None, ctypes.byref(info))
        return {"kernel": info.kernel.decode(), "grid": int(info.grid), "block": int(info.block),
                "smem_bytes": int(info.smem_bytes), "peek_bits": int(info.peek_bits),
                "table_copies": int(info.table_copies), "thread_blocks": int(info.thread_blocks)}

    def views(self, flat: torch.Tensor) -> list[torch.Tensor]:
        """Per-matrix views of a decompressed flat buffer."""
        out = []
        for k, shape in enumerate(self.shapes):
            a, b = int(self.header.seg_elem_off[k]), int(self.header.seg_elem_off[k + 1])
            out.append(flat[a:b].view(shape))
        return out


def code_lengths(hist: np.ndarray, max_code_len: int = 32) -> np.ndarray:
    """The library's host code builder (package-merge), for tests."""
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    out = np.zeros(256, dtype=np.uint8)
    B.call("df11_code_lengths", _np_ptr(h), max_code_len, _np_ptr(out))
    return out


def make_header(code_len: np.ndarray, n_elems: int, total_bits: int,
                threads_per_block: int = DEFAULT_THREADS_PER_BLOCK,
                max_code_len: int = 32, seg_counts=None) -> B.Header:
    hdr = B.Header()
    ln = np.ascontiguousarray(code_len, dtype=np.uint8)
    if seg_counts is None:
        seg_counts = [n_elems]
    counts = np.ascontiguousarray(seg_counts, dtype=np.uint64)
    B.call("df11_header_init", ctypes.byref(hdr), _np_ptr(ln), n_elems, total_bits, threads_per_block,
           max_code_len, _np_ptr(counts), len(counts))
    return hdr


def build_lut(header: B.Header) -> np.ndarray:
    out = np.zeros(int(header.bytes_lut), dtype=np.uint8)
    B.call("df11_build_lut", ctypes.byref(header), _np_ptr(out), out.size)
    return out


def workspace_bytes(n_elems: int) -> int:
    v = ctypes.c_uint64()
    B.call("df11_compress_workspace_size", n_elems, ctypes.byref(v))
    return int(v.value)


def _as_segments(tensors, dtype=torch.bfloat16):
    if isinstance(tensors, torch.Tensor):
        tensors = [tensors]
    segs = []
    for t in tensors:
        if t.dtype != dtype:
            raise TypeError(f"expected {dtype} tensors, got {t.dtype}")
        if not t.is_cuda:
            raise ValueError("compress expects CUDA tensors")
        segs.append(t.contiguous())
    return segs


def compress(tensors, names=None, threads_per_block: int = DEFAULT_THREADS_PER_BLOCK, max_code_len: int = 32,
             stream=None) -> CompressedStream:
    """Compress one BF16 tensor, or a list (a transformer block) into one
    stream with a shared code table: histogram kernel, host code builder,
    encode kernel (the decode tables are built on the host while it runs).
    Synchronises the stream once for the histogram readback, and again at
    the end, before the workspace is released."""
    segs = _as_segments(tensors)
    device = segs[0].device
    n = sum(t.numel() for t in segs)
    ws = torch.empty(max(workspace_bytes(n), 16), dtype=torch.uint8, device=device)
    ptrs = (ctypes.c_void_p * len(segs))(*[int(t.data_ptr()) for t in segs])
    counts = (ctypes.c_uint64 * len(segs))(*[t.numel() for t in segs])
    hdr = B.Header()
    sh = _stream_handle(stream)
    B.call("df11_compress_plan", ptrs, counts, len(segs), threads_per_block, max_code_len, _ptr(ws),
           ws.numel(), ctypes.byref(hdr), sh)
    exp = torch.empty(int(hdr.bytes_exp), dtype=torch.uint8, device=device)
    sm = torch.empty(int(hdr.bytes_sm) or 16, dtype=torch.uint8, device=device)
    gaps = torch.empty(int(hdr.bytes_gaps), dtype=torch.uint8, device=device)
    off = torch.empty(int(hdr.n_blocks) + 1, dtype=torch.int32, device=device)
    lut = torch.empty(int(hdr.bytes_lut), dtype=torch.uint8, device=device)
    B.call("df11_compress_encode", ptrs, ctypes.byref(hdr), _ptr(ws), ws.numel(), _ptr(exp), _ptr(sm),
           _ptr(gaps), _ptr(off), _ptr(lut), sh)
    # keep the workspace alive until the queued kernels have consumed it
    (stream or torch.cuda.current_stream()).synchronize()
    return CompressedStream(hdr, exp, sm, gaps, off, lut,
                            names=list(names) if names else [f"t{k}" for k in range(len(segs))],
                            shapes=[tuple(t.shape) for t in segs])


def from_arrays(code_len: np.ndarray, n_elems: int, total_bits: int, threads_per_block: int,
                exp: np.ndarray, sm: np.ndarray | None, gaps: np.ndarray, block_off: np.ndarray,
                max_code_len: int = 32, seg_counts=None, shapes=None, device="cuda",
                symbols: str = "bf16") -> CompressedStream:
    """Upload a stream made elsewhere (another encoder, a file); streams of
    8-bit symbols (symbols="u8") have no sm array."""
    hdr = make_header(code_len, n_elems, total_bits, threads_per_block, max_code_len, seg_counts)
    if symbols == "u8":
        sm = np.zeros(0, dtype=np.uint8)
    arrays = [("exp", exp, hdr.bytes_exp), ("gaps", gaps, hdr.bytes_gaps), ("block_off", block_off, hdr.n_blocks + 1)]
    if symbols == "bf16":
        arrays.append(("sm", sm, hdr.bytes_sm))
    for name, arr, need in arrays:
        if arr.size < need:
            raise ValueError(f"{name}: {arr.size} entries, header needs {need}")
    lut = build_lut(hdr)

    def up(a, dtype=torch.uint8):
        a = np.ascontiguousarray(a)
        if a.size == 0:
            return torch.zeros(16, dtype=dtype, device=device)
        return torch.from_numpy(a.view(np.int32) if dtype == torch.int32 else a).to(device)

    shapes = shapes or [(int(c),) for c in (seg_counts or [n_elems])]
    return CompressedStream(hdr, up(exp), up(sm), up(gaps),
                            up(np.ascontiguousarray(block_off, dtype=np.uint32), torch.int32), up(lut),
                            names=[f"t{k}" for k in range(len(shapes))], shapes=shapes, symbols=symbols)


def to_host(cs: CompressedStream) -> dict:
    """The stream's arrays as numpy (for another decoder)."""
    h = cs.header
    return dict(code_len=cs.code_len, n_elems=int(h.n_elems), total_bits=int(h.total_bits),
                threads_per_block=int(h.threads_per_block), n_threads=int(h.n_threads),
                n_blocks=int(h.n_blocks),
                exp=cs.exp.cpu().numpy()[: int(h.bytes_exp)],
                sm=cs.sm.cpu().numpy()[: int(h.bytes_sm)] if cs.symbols == "bf16" else np.zeros(0, np.uint8),
                gaps=cs.gaps.cpu().numpy()[: int(h.bytes_gaps)],
                block_off=cs.block_off.cpu().numpy().view(np.uint32)[: int(h.n_blocks) + 1])


def decode_options(peek_bits: int = 0, max_sms: int = 0, max_warps_per_cta: int = 0, ctas: int = 0,
                   block_begin: int = 0, block_end: int = 0, early_staging: bool = False):
    """df11_decode_options (all zero: the library's defaults; a block range
    decodes only those thread blocks, as decompress_blocks).  early_staging:
    the caller states that the kernel launched just before the decode on its
    stream writes none of the stream's arrays (e.g. the previous block's
    decode, or a consumer GEMM), so the decode stages its tables and first
    loads while that kernel finishes."""
    return B.DecodeOptions(peek_bits, max_sms, max_warps_per_cta, ctas, block_begin, block_end,
                           1 if early_staging else 0, 0)


def decompress(cs: CompressedStream, out: torch.Tensor | None = None, status: torch.Tensor | None = None,
               stream=None, max_sms: int | None = None, options=None) -> torch.Tensor:
    """One kernel launch rebuilding all n_elems BF16 values of the stream.
    Asynchronous; `out` (bfloat16, n_elems, contiguous) may be reused across
    calls.  `status` (int32 device word, zeroed by the caller) receives
    DF11_ERR_CORRUPT if the stream disagrees with its metadata.  `max_sms`
    caps the SMs the decode occupies (df11_decompress_sms), leaving the rest
    to kernels on other streams; `options` (decode_options) selects the
    table width and launch shape (df11_decompress_opts)."""
    n = cs.n_elems
    if out is None:
        out = torch.empty(max(n, 1), dtype=torch.bfloat16, device=cs.exp.device)[:n]
    if out.dtype != torch.bfloat16 or not out.is_contiguous() or out.numel() < n:
        raise ValueError("out must be a contiguous bfloat16 tensor with n_elems elements")
    st = _ptr(status) if status is not None else ctypes.c_void_p(0)
    args = (ctypes.byref(cs.header), _ptr(cs.exp), _ptr(cs.sm), _ptr(cs.gaps), _ptr(cs.block_off),
            _ptr(cs.lut), _ptr(out))
    if options is not None:
        B.call("df11_decompress_opts", *args, 0, ctypes.byref(options), st, _stream_handle(stream))
    elif max_sms is None:
        B.call("df11_decompress", *args, st, _stream_handle(stream))
    else:
        B.call("df11_decompress_sms", *args, st, ctypes.c_uint32(max_sms), _stream_handle(stream))
    return out


def decompress_blocks(cs: CompressedStream, block_begin: int, block_end: int, out: torch.Tensor,
                      status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Decode thread blocks [block_begin, block_end) of the stream only
    (df11_decompress_blocks, or df11_decompress_u8_blocks for 8-bit symbols):
    writes output elements [off[block_begin], off[block_end]) of `out`, the
    whole stream's output buffer, and leaves the rest as it is.  Reads only
    the bytes `piece_ranges` lists.  Asynchronous."""
    u8 = cs.symbols == "u8"
    dtype = torch.uint8 if u8 else torch.bfloat16
    if out.dtype != dtype or not out.is_contiguous() or out.numel() < cs.n_elems:
        raise ValueError(f"out must be a contiguous {dtype} tensor with n_elems elements")
    st = _ptr(status) if status is not None else ctypes.c_void_p(0)
    b0, b1 = ctypes.c_uint64(block_begin), ctypes.c_uint64(block_end)
    if u8:
        B.call("df11_decompress_u8_blocks", ctypes.byref(cs.header), _ptr(cs.exp), _ptr(cs.gaps),
               _ptr(cs.block_off), _ptr(cs.lut), _ptr(out), b0, b1, st, _stream_handle(stream))
    else:
        B.call("df11_decompress_blocks", ctypes.byref(cs.header), _ptr(cs.exp), _ptr(cs.sm), _ptr(cs.gaps),
               _ptr(cs.block_off), _ptr(cs.lut), _ptr(out), b0, b1, st, _stream_handle(stream))
    return out


def piece_ranges(header, block_off, b0: int, b1: int, u8: bool = False) -> dict[str, tuple[int, int]]:
    """Byte ranges [lo, hi) of each stream array that decoding thread blocks
    [b0, b1) reads (the contract of df11_decompress_blocks): EncodedExponent
    from the piece's first window to 16 bytes past its last, the gap fields
    of its windows plus one 8-byte lookahead, block offsets b0..b1, and the
    sign+mantissa bytes of its elements widened to 128 bytes below and 16
    above; each clipped to the array's size.  `block_off` is the host copy of
    the offsets (any integer sequence)."""
    T = int(header.threads_per_block)
    lo_e, hi_e = int(block_off[b0]), int(block_off[b1])
    r = {
        "exp": (8 * T * b0, min(8 * T * b1 + 16, int(header.bytes_exp))),
        "gaps": ((5 * T * b0) // 8, min((5 * T * b1 + 7) // 8 + 8, int(header.bytes_gaps))),
        "block_off": (4 * b0, 4 * (b1 + 1)),
    }
    if not u8:
        r["sm"] = (lo_e & ~127, min((hi_e + 15) & ~15, int(header.bytes_sm)))
    return r


class HostStream:
    """A stream kept in pinned host memory, decompressed end to end: copy the
    compressed arrays to the device, decode, copy the result (BF16, or bytes
    for a stream of 8-bit symbols) back.

    `run` splits the stream into pieces of whole thread blocks and pipelines
    them over three CUDA streams: the copy of piece i+1 to the device, the
    decode of piece i (on the caller's stream) and the copy of piece i-1
    back run at the same time, so the two directions of the host link
    overlap each other and the decode."""

    # output bytes per piece when `pieces` is not given: on a Llama-3.1-8B block
    # (436 MB out) 8 pieces came within 5% of the host link's bidirectional
    # limit, while every piece also costs host-side launch and copy calls
    # (36 pieces were 17% slower than 8, 128 pieces 34%)
    PIECE_OUT_BYTES = 48 << 20
    MAX_PIECES = 16

    def __init__(self, cs: CompressedStream):
        self.header = cs.header
        self.u8 = cs.symbols == "u8"
        keys = ("exp", "gaps", "block_off", "lut") if self.u8 else ("exp", "sm", "gaps", "block_off", "lut")
        self.host = {k: getattr(cs, k).cpu().pin_memory() for k in keys}
        dev = cs.exp.device
        self.dev = {k: torch.empty_like(v, device=dev) for k, v in self.host.items()}
        self.dev_stream = CompressedStream(cs.header, self.dev["exp"], self.dev.get("sm", cs.sm), self.dev["gaps"],
                                           self.dev["block_off"], self.dev["lut"], cs.names, cs.shapes,
                                           symbols=cs.symbols)
        dtype = torch.uint8 if self.u8 else torch.bfloat16
        n = cs.n_elems
        self.out_dev = torch.empty(max(n, 16), dtype=dtype, device=dev)[:n]
        self.out_host = torch.empty(max(n, 16), dtype=dtype).pin_memory()[:n]
        self.off = self.host["block_off"].numpy().view(np.uint32)
        self._side = None
        self.last_h2d_bytes = 0

    def h2d_bytes(self) -> int:
        """Bytes the last `run` copied to the device (every array once, plus
        the few bytes pieces share); before any run, the arrays' sizes."""
        return self.last_h2d_bytes or sum(v.numel() * v.element_size() for v in self.host.values())

    def d2h_bytes(self) -> int:
        return self.out_host.element_size() * int(self.header.n_elems)

    def default_pieces(self) -> int:
        return max(1, min(self.MAX_PIECES, self.d2h_bytes() // self.PIECE_OUT_BYTES))

    def run(self, stream=None, pieces: int | None = None) -> torch.Tensor:
        s = stream or torch.cuda.current_stream()
        nb = int(self.header.n_blocks)
        n_pieces = max(1, min(self.default_pieces() if pieces is None else int(pieces), nb))
        decode = decompress_u8 if self.u8 else decompress
        if n_pieces == 1:
            with torch.cuda.stream(s):
                for k, v in self.host.items():
                    self.dev[k].copy_(v, non_blocking=True)
                decode(self.dev_stream, self.out_dev, stream=s)
                self.out_host.copy_(self.out_dev, non_blocking=True)
            self.last_h2d_bytes = sum(v.numel() * v.element_size() for v in self.host.values())
            return self.out_host
        if self._side is None:
            dev = self.out_dev.device
            self._side = (torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev))
        s_in, s_out = self._side
        # the buffers may still be in use by work already queued on the caller's stream
        s_in.wait_stream(s)
        s_out.wait_stream(s)
        h2d = 0
        with torch.cuda.stream(s_in):
            self.dev["lut"].copy_(self.host["lut"], non_blocking=True)
            h2d += self.host["lut"].numel()
        bounds = [nb * i // n_pieces for i in range(n_pieces + 1)]
        for i in range(n_pieces):
            b0, b1 = bounds[i], bounds[i + 1]
            with torch.cuda.stream(s_in):
                for k, (lo, hi) in piece_ranges(self.header, self.off, b0, b1, self.u8).items():
                    src, dst = self.host[k], self.dev[k]
                    if k == "block_off":  # int32 entries
                        lo, hi = lo // 4, hi // 4
                    dst[lo:hi].copy_(src[lo:hi], non_blocking=True)
                    h2d += (hi - lo) * src.element_size()
            ready = torch.cuda.Event()
            ready.record(s_in)
            s.wait_event(ready)
            decompress_blocks(self.dev_stream, b0, b1, self.out_dev, stream=s)
            done = torch.cuda.Event()
            done.record(s)
            s_out.wait_event(done)
            e0, e1 = int(self.off[b0]), int(self.off[b1])
            with torch.cuda.stream(s_out):
                self.out_host[e0:e1].copy_(self.out_dev[e0:e1], non_blocking=True)
        s.wait_stream(s_out)
        self.last_h2d_bytes = h2d
        return self.out_host


def compress_u8(tensors, names=None, threads_per_block: int = DEFAULT_THREADS_PER_BLOCK, max_code_len: int = 32,
                stream=None) -> CompressedStream:
    """Compress one uint8 tensor (e.g. per-tensor quantized weights), or a
    list, coding each byte whole with one shared table; no side array.  T = 128
    falls back to T = 32 when the code has a 1-bit symbol (the decoder with
    four windows per lane needs codes of 2 bits or more)."""
    segs = _as_segments(tensors, torch.uint8)
    device = segs[0].device
    n = sum(t.numel() for t in segs)
    ws = torch.empty(max(workspace_bytes(n), 16), dtype=torch.uint8, device=device)
    ptrs = (ctypes.c_void_p * len(segs))(*[int(t.data_ptr()) for t in segs])
    counts = (ctypes.c_uint64 * len(segs))(*[t.numel() for t in segs])
    hdr = B.Header()
    sh = _stream_handle(stream)
    B.call("df11_compress_plan_u8", ptrs, counts, len(segs), threads_per_block, max_code_len, _ptr(ws),
           ws.numel(), ctypes.byref(hdr), sh)
    ln = np.frombuffer(bytes(hdr.code_len), dtype=np.uint8)
    if threads_per_block == 128 and n and ln[ln > 0].min() == 1:
        token = hdr.plan_token  # the plan's per-range histograms do not depend on T
        hdr = make_header(ln, int(hdr.n_elems), int(hdr.total_bits), 32, max_code_len,
                          [t.numel() for t in segs])
        hdr.plan_token = token
    exp = torch.empty(int(hdr.bytes_exp), dtype=torch.uint8, device=device)
    gaps = torch.empty(int(hdr.bytes_gaps), dtype=torch.uint8, device=device)
    off = torch.empty(int(hdr.n_blocks) + 1, dtype=torch.int32, device=device)
    lut = torch.empty(int(hdr.bytes_lut), dtype=torch.uint8, device=device)
    B.call("df11_compress_encode_u8", ptrs, ctypes.byref(hdr), _ptr(ws), ws.numel(), _ptr(exp), _ptr(gaps),
           _ptr(off), _ptr(lut), sh)
    (stream or torch.cuda.current_stream()).synchronize()
    return CompressedStream(hdr, exp, torch.zeros(16, dtype=torch.uint8, device=device), gaps, off, lut,
                            names=list(names) if names else [f"t{k}" for k in range(len(segs))],
                            shapes=[tuple(t.shape) for t in segs], symbols="u8")


def decompress_u8(cs: CompressedStream, out: torch.Tensor | None = None, status: torch.Tensor | None = None,
                  stream=None, options=None) -> torch.Tensor:
    """One kernel launch rebuilding all n_elems bytes of a stream of 8-bit
    symbols.  Asynchronous; `out` (uint8, n_elems, contiguous, 16-byte
    aligned) may be reused; `options` as for decompress."""
    if cs.symbols != "u8":
        raise ValueError("decompress_u8 takes streams of 8-bit symbols (compress_u8)")
    n = cs.n_elems
    if out is None:
        out = torch.empty(max(n, 16), dtype=torch.uint8, device=cs.exp.device)[:n]
    if out.dtype != torch.uint8 or not out.is_contiguous() or out.numel() < n:
        raise ValueError("out must be a contiguous uint8 tensor with n_elems elements")
    st = _ptr(status) if status is not None else ctypes.c_void_p(0)
    if options is not None:
        B.call("df11_decompress_opts", ctypes.byref(cs.header), _ptr(cs.exp), ctypes.c_void_p(0), _ptr(cs.gaps),
               _ptr(cs.block_off), _ptr(cs.lut), _ptr(out), 1, ctypes.byref(options), st, _stream_handle(stream))
    else:
        B.call("df11_decompress_u8", ctypes.byref(cs.header), _ptr(cs.exp), _ptr(cs.gaps), _ptr(cs.block_off),
               _ptr(cs.lut), _ptr(out), st, _stream_handle(stream))
    return out


IND_CHUNK = 64  # elements per independently decodable chunk


@dataclass
class ChunkedStream:
    """The independent-chunk variant of a stream: EncodedExponent,
    PackedSignMantissa and the decode tables as in a DF11 stream, and the
    start bit of every IND_CHUNK elements (then total_bits) instead of Gaps
    and block offsets."""
    header: B.Header
    exp: torch.Tensor
    sm: torch.Tensor
    chunk_bit: torch.Tensor  # int32 storage of uint32 start bits
    lut: torch.Tensor
    names: list = field(default_factory=list)
    shapes: list = field(default_factory=list)

    @property
    def n_elems(self) -> int:
        return int(self.header.n_elems)

    @property
    def n_chunks(self) -> int:
        return (self.n_elems + IND_CHUNK - 1) // IND_CHUNK

    def compressed_bytes(self) -> int:
        """Code bits, one byte per element, the chunk table and the 256-byte
        code-length table."""
        h = self.header
        return (h.total_bits + 7) // 8 + h.n_elems + 4 * (self.n_chunks + 1) + 256

    def read_bytes(self) -> int:
        h = self.header
        return (h.total_bits + 7) // 8 + h.n_elems + 4 * (self.n_chunks + 1)

    def views(self, flat: torch.Tensor) -> list[torch.Tensor]:
        out = []
        for k, shape in enumerate(self.shapes):
            a, b = int(self.header.seg_elem_off[k]), int(self.header.seg_elem_off[k + 1])
            out.append(flat[a:b].view(shape))
        return out


def compress_chunked(tensors, names=None, max_code_len: int = 32, stream=None) -> ChunkedStream:
    """Compress BF16 tensors into the independent-chunk variant: the same code
    and bit stream as `compress`, with a chunk table for the decoder."""
    segs = _as_segments(tensors)
    device = segs[0].device
    n = sum(t.numel() for t in segs)
    ws = torch.empty(max(workspace_bytes(n), 16), dtype=torch.uint8, device=device)
    ptrs = (ctypes.c_void_p * len(segs))(*[int(t.data_ptr()) for t in segs])
    counts = (ctypes.c_uint64 * len(segs))(*[t.numel() for t in segs])
    hdr = B.Header()
    sh = _stream_handle(stream)
    B.call("df11_compress_plan", ptrs, counts, len(segs), DEFAULT_THREADS_PER_BLOCK, max_code_len, _ptr(ws),
           ws.numel(), ctypes.byref(hdr), sh)
    exp = torch.empty(int(hdr.bytes_exp), dtype=torch.uint8, device=device)
    sm = torch.empty(int(hdr.bytes_sm) or 16, dtype=torch.uint8, device=device)
    chunk_bit = torch.empty(max((n + IND_CHUNK - 1) // IND_CHUNK + 1, 4), dtype=torch.int32, device=device)
    lut = torch.empty(int(hdr.bytes_lut), dtype=torch.uint8, device=device)
    B.call("df11_compress_encode_chunked", ptrs, ctypes.byref(hdr), _ptr(ws), ws.numel(), _ptr(exp), _ptr(sm),
           _ptr(chunk_bit), _ptr(lut), sh)
    (stream or torch.cuda.current_stream()).synchronize()
    return ChunkedStream(hdr, exp, sm, chunk_bit, lut,
                         names=list(names) if names else [f"t{k}" for k in range(len(segs))],
                         shapes=[tuple(t.shape) for t in segs])


def chunked_from_arrays(code_len: np.ndarray, n_elems: int, total_bits: int, exp: np.ndarray, sm: np.ndarray,
                        chunk_bit: np.ndarray, max_code_len: int = 32, seg_counts=None, shapes=None,
                        device="cuda") -> ChunkedStream:
    """Upload an independent-chunk stream made elsewhere."""
    hdr = make_header(code_len, n_elems, total_bits, DEFAULT_THREADS_PER_BLOCK, max_code_len, seg_counts)
    lut = build_lut(hdr)
    up = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    cb = np.ascontiguousarray(chunk_bit, dtype=np.uint32).view(np.int32)
    shapes = shapes or [(int(c),) for c in (seg_counts or [n_elems])]
    return ChunkedStream(hdr, up(exp), up(sm), up(cb), up(lut), names=[f"t{k}" for k in range(len(shapes))],
                         shapes=shapes)


def decompress_chunked(cs: ChunkedStream, out: torch.Tensor | None = None, status: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """One launch of the independent-chunk decoder; asynchronous."""
    n = cs.n_elems
    if out is None:
        out = torch.empty(max(n, 8), dtype=torch.bfloat16, device=cs.exp.device)[:n]
    if out.dtype != torch.bfloat16 or not out.is_contiguous() or out.numel() < n:
        raise ValueError("out must be a contiguous bfloat16 tensor with n_elems elements")
    B.call("df11_decompress_chunked", ctypes.byref(cs.header), _ptr(cs.exp), _ptr(cs.sm), _ptr(cs.chunk_bit),
           _ptr(cs.lut), _ptr(out), _ptr(status) if status is not None else ctypes.c_void_p(0),
           _stream_handle(stream))
    return out
