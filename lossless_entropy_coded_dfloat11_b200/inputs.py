"""Seeded synthetic BF16 workloads.

This module only makes inputs: it holds none of the codec's arithmetic and is
the one piece the tests, the benchmark and the oracle checks share.  Trained
LLM weights are not available, so Gaussian stand-ins with the shapes and
scales of real checkpoints take their place:

* ``matrix_1k``      1024x1024, N(0, 0.02), seed 1.
* ``matrix_outliers`` 14336x4096, N(0, 0.02), seed 2; 0.1% of the entries
  (a seeded permutation) replaced by Laplace(0, 0.5) draws and the next 0.01%
  set to +0.0 (long codes, zero exponent).
* ``llama_block``    one transformer block in the Llama-3.1 layout
  (attn_norm, q, k, v, o, mlp_norm, gate, up, down), projections
  N(0, 1/sqrt(fan_in)) with fan_in the second dimension of the out x in
  shape, RMSNorm vectors N(1, 0.05); 8B shapes (hidden 4096, intermediate
  14336, 8 KV heads x 128) or 70B shapes (hidden 8192, intermediate 28672).
* ``edge_case``      n elements whose exponent is uniform over 0..254, 99.9%
  one value (120), or Zipf(s=1.2) over 255 ranks mapped to exponents by a
  seeded permutation; sign and mantissa are a uniform random byte.
* ``all_patterns``   every one of the 65536 BF16 bit patterns, shuffled.
* ``fibonacci``      exponent counts 1, 1, 2, 3, 5, ... (34 values): the
  unrestricted Huffman tree is 33 deep, so a 32-bit length limit binds.

Values are drawn in fp32 on a seeded ``torch.Generator`` and rounded to BF16
(round to nearest even).  ``device="cuda"`` draws on the GPU instead (other
numbers, same distribution), which the benchmark uses to build its large
inputs quickly.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

SIGMA_DEFAULT = 0.02


@dataclass
class Workload:
    name: str
    names: list[str]          # one per matrix / vector
    tensors: list[torch.Tensor]  # bfloat16 (uint8 for 8-bit symbol workloads), 1-D or 2-D, same device

    @property
    def n_elems(self) -> int:
        return sum(t.numel() for t in self.tensors)

    def flat_u16(self) -> np.ndarray:
        """All segments concatenated, as uint16 bit patterns on the host."""
        parts = [t.detach().reshape(-1).view(torch.int16).cpu().numpy().view(np.uint16)
                 for t in self.tensors]
        if not parts:
            return np.zeros(0, dtype=np.uint16)
        return np.concatenate(parts)


def _gen(seed: int, device: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def gaussian(shape, sigma: float, seed: int, mean: float = 0.0, device: str = "cpu") -> torch.Tensor:
    g = _gen(seed, device)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if sigma != 1.0:
        x.mul_(sigma)
    if mean != 0.0:
        x.add_(mean)
    return x.to(torch.bfloat16)


def matrix_1k(device: str = "cpu") -> Workload:
    return Workload("matrix_1k", ["w"], [gaussian((1024, 1024), SIGMA_DEFAULT, 1, device=device)])


def matrix_outliers(rows: int = 14336, cols: int = 4096, seed: int = 2,
                    device: str = "cpu") -> Workload:
    g = _gen(seed, device)
    n = rows * cols
    x = torch.randn(n, generator=g, device=device, dtype=torch.float32).mul_(SIGMA_DEFAULT)
    n_out = n // 1000          # 0.1 %
    n_zero = n // 10000        # 0.01 %
    perm = torch.randperm(n, generator=g, device=device)
    pos_out = perm[:n_out]
    pos_zero = perm[n_out:n_out + n_zero]
    # Laplace(0, b) by inverting its CDF on u ~ U(-1/2, 1/2)
    u = torch.rand(n_out, generator=g, device=device, dtype=torch.float64) - 0.5
    lap = -0.5 * torch.sign(u) * torch.log1p(-2.0 * u.abs())
    x[pos_out] = lap.to(torch.float32)
    x[pos_zero] = 0.0
    return Workload("matrix_outliers", ["w"], [x.to(torch.bfloat16).reshape(rows, cols)])


LLAMA_8B = dict(hidden=4096, intermediate=14336, kv=1024)
LLAMA_70B = dict(hidden=8192, intermediate=28672, kv=1024)
BLOCK_ORDER = ["attn_norm", "q", "k", "v", "o", "mlp_norm", "gate", "up", "down"]


def block_shapes(hidden: int, intermediate: int, kv: int) -> list[tuple[str, tuple[int, ...]]]:
    h, f = hidden, intermediate
    shapes = {"attn_norm": (h,), "q": (h, h), "k": (kv, h), "v": (kv, h), "o": (h, h),
              "mlp_norm": (h,), "gate": (f, h), "up": (f, h), "down": (h, f)}
    return [(name, shapes[name]) for name in BLOCK_ORDER]


def llama_block(cfg: dict = LLAMA_8B, seed_base: int = 3, device: str = "cpu") -> Workload:
    """Projection weights N(0, 1/sqrt(fan_in)); norm weights N(1, 0.05).
    Tensor k of the block is drawn with seed ``seed_base + k``."""
    names, tensors = [], []
    for k, (name, shape) in enumerate(block_shapes(**cfg)):
        seed = seed_base + k
        if len(shape) == 1:
            t = gaussian(shape, 0.05, seed, mean=1.0, device=device)
        else:
            t = gaussian(shape, 1.0 / math.sqrt(shape[1]), seed, device=device)
        names.append(name)
        tensors.append(t)
    return Workload("llama3.1-8b-block" if cfg == LLAMA_8B else "llama3.1-70b-block", names, tensors)


def llama70b_block(block: int, device: str = "cpu") -> Workload:
    """Block ``block`` (0..7) of the 70B-shaped set: seeds 100 + 16*block + k."""
    return llama_block(LLAMA_70B, seed_base=100 + 16 * block, device=device)


EDGE_SIZES = [1, 2, 3, 7, 8, 9, 31, 33, 63, 65, 127, 255, 257, 1023, 4097, 65537,
              2 ** 20 + 7, 2 ** 24 + 3, 2 ** 26 + 13]
EDGE_DISTS = ["uniform", "one_value", "zipf"]


def _bf16_from_fields(exponent: torch.Tensor, sign_mant: torch.Tensor) -> torch.Tensor:
    """Assemble BF16 numbers from an 8-bit biased exponent and a random
    sign/mantissa byte (bit 7 -> sign, bits 6..0 -> mantissa)."""
    e = exponent.to(torch.int32)
    b = sign_mant.to(torch.int32)
    bits = ((b >> 7) << 15) | (e << 7) | (b & 0x7F)
    u16 = bits.numpy().astype(np.uint16)
    return torch.from_numpy(u16.view(np.int16)).view(torch.bfloat16)


def edge_case(n: int, dist: str, seed: int) -> Workload:
    g = _gen(seed, "cpu")
    if dist == "uniform":
        e = torch.randint(0, 255, (n,), generator=g)
    elif dist == "one_value":
        e = torch.full((n,), 120, dtype=torch.int64)
        rare = torch.rand(n, generator=g) < 0.001
        k = int(rare.sum())
        other = torch.randint(0, 254, (k,), generator=g)
        other = other + (other >= 120).to(other.dtype)   # any value but 120
        e[rare] = other
    elif dist == "zipf":
        ranks = torch.arange(1, 256, dtype=torch.float64)
        p = ranks.pow(-1.2)
        cdf = torch.cumsum(p / p.sum(), 0)
        u = torch.rand(n, generator=g, dtype=torch.float64)
        r = torch.searchsorted(cdf, u).clamp_(max=254)
        perm = torch.randperm(255, generator=g)
        e = perm[r]
    else:
        raise ValueError(dist)
    sm = torch.randint(0, 256, (n,), generator=g)
    return Workload(f"edge_{dist}_{n}", ["x"], [_bf16_from_fields(e, sm)])


def all_patterns(seed: int = 7) -> Workload:
    g = _gen(seed, "cpu")
    bits = torch.randperm(65536, generator=g).numpy().astype(np.uint16)
    return Workload("all_patterns", ["x"], [torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)])


def fibonacci(k: int = 34, seed: int = 11, first_exponent: int = 100) -> Workload:
    """Exponent value first_exponent + j occurs F_(j+1) times (F_1 = F_2 = 1),
    j = 0..k-1, in a seeded random order."""
    fib = [1, 1]
    while len(fib) < k:
        fib.append(fib[-1] + fib[-2])
    e = torch.cat([torch.full((c,), first_exponent + j, dtype=torch.int64) for j, c in enumerate(fib[:k])])
    g = _gen(seed, "cpu")
    e = e[torch.randperm(e.numel(), generator=g)]
    sm = torch.randint(0, 256, (e.numel(),), generator=g)
    return Workload(f"fibonacci_{k}", ["x"], [_bf16_from_fields(e, sm)])


# --------------------------------------------------------------------------- #
# 8-bit symbol streams                                                        #
# --------------------------------------------------------------------------- #
def quantize_u8(t: torch.Tensor) -> torch.Tensor:
    """Per-tensor asymmetric 8-bit quantisation: the tensor's range [min, max]
    mapped onto 0..255 (round to nearest).  Generates the kind of integer
    symbols an entropy coder of quantized weights sees; the codec itself
    takes the bytes as they are."""
    x = t.float()
    lo, hi = x.min(), x.max()
    scale = (hi - lo).clamp_min(1e-30) / 255.0
    return torch.round((x - lo) / scale).clamp_(0, 255).to(torch.uint8)


def quantize_u4(t: torch.Tensor) -> torch.Tensor:
    """Per-tensor asymmetric 4-bit quantisation onto 0..15 (round to nearest),
    one value per byte: the 16-symbol alphabet of uint4 weights, coded whole
    by the same 8-bit-symbol streams."""
    x = t.float()
    lo, hi = x.min(), x.max()
    scale = (hi - lo).clamp_min(1e-30) / 15.0
    return torch.round((x - lo) / scale).clamp_(0, 15).to(torch.uint8)


def llama_block_u4(cfg: dict = LLAMA_8B, seed_base: int = 3, device: str = "cpu") -> Workload:
    """The matrices of `llama_block` quantized per tensor to 4 bits, one value
    per byte."""
    w = llama_block(cfg, seed_base, device)
    return Workload(w.name + "-u4", list(w.names), [quantize_u4(t) for t in w.tensors])


def llama_block_u8(cfg: dict = LLAMA_8B, seed_base: int = 3, device: str = "cpu") -> Workload:
    """The matrices of `llama_block` quantized per tensor to uint8."""
    w = llama_block(cfg, seed_base, device)
    return Workload(w.name + "-u8", list(w.names), [quantize_u8(t) for t in w.tensors])


def edge_case_u8(n: int, dist: str, seed: int) -> Workload:
    """n bytes with the symbol distribution of `edge_case` (uniform over
    0..254, 99.9% one value, Zipf over a permuted alphabet)."""
    w = edge_case(n, dist, seed)
    x = w.tensors[0].view(torch.int16).to(torch.int32)
    return Workload(f"edge_u8_{dist}_{n}", ["x"], [((x >> 7) & 0xFF).to(torch.uint8)])
