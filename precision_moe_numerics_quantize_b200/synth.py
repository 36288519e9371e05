"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module holds no arithmetic of the quantization method. It only produces
input tensors. The generator is counter-based: element n of stream (seed, tag)
depends only on (seed, tag, n), so a CPU caller can produce any slice of a
tensor (for example one expert's weights) and get exactly the bits that the
device-side generator writes for the whole tensor.

Distribution. An approximately normal value is the centred sum of eight 16-bit
uniforms (Irwin-Hall, n = 8; bounded at about 4.9 sigma), scaled to the wanted
standard deviation with one fp32 multiply and rounded to bf16 (nearest, ties to
even). Every step is integer arithmetic or a single IEEE fp32 operation, so
numpy and torch (CPU or CUDA) agree bit for bit. A heavy-tailed variant
multiplies such a normal by 2^k with P(k >= j) = 8^-j, so its tail falls like
|x|^-3 (the tail of a Student-t with 3 degrees of freedom) using only exact
products.

Integer hashing uses 32-bit words carried in int64 with explicit masking; the
32x32-bit products are split into 16-bit halves so that nothing overflows int64.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

M32 = 0xFFFFFFFF
_IH_N = 8
_IH_CENTER = _IH_N * 65535 // 2  # 262140, exact because 8 * 65535 is even
_IH_SIGMA = math.sqrt(_IH_N * (65536.0 ** 2 - 1.0) / 12.0)


# --------------------------------------------------------------------------
# integer hash (lowbias32 mixing) in a backend-neutral form
# --------------------------------------------------------------------------

def _mul32(x, c: int):
    lo = (x & 0xFFFF) * c
    hi = (((x >> 16) * (c & 0xFFFF)) & 0xFFFF) << 16
    return (lo + hi) & M32


def _mix32(x):
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def _mix32_int(x: int) -> int:
    x &= M32
    x ^= x >> 16
    x = (x * 0x7FEB352D) & M32
    x ^= x >> 15
    x = (x * 0x846CA68B) & M32
    x ^= x >> 16
    return x


def _stream_keys(seed: int, tag: int):
    base = _mix32_int(_mix32_int(seed & M32) ^ _mix32_int((seed >> 32) ^ (tag * 0x9E3779B9)))
    return [_mix32_int(base ^ (j * 0x85EBCA6B + 0x27D4EB2F)) for j in range(_IH_N // 2)]


def _ih_sum(n, keys):
    """Centred sum of eight 16-bit uniforms for element indices n (int64)."""
    n_lo = n & M32
    n_hi = n >> 32
    z = None
    for kj in keys:
        h = _mix32(_mix32(n_lo ^ kj) ^ n_hi)
        part = (h & 0xFFFF) + (h >> 16)
        z = part if z is None else z + part
    return z - _IH_CENTER


def _scale_const(std: float) -> np.float32:
    return np.float32(std / _IH_SIGMA)


# --------------------------------------------------------------------------
# bf16 rounding of fp32 values (nearest, ties to even), numpy side
# --------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = np.isnan(x)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    r = r.astype(np.uint16)
    r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------
# numpy generators (host)
# --------------------------------------------------------------------------

def normal_f32_np(seed: int, tag: int, start: int, count: int, std: float) -> np.ndarray:
    n = np.arange(start, start + count, dtype=np.int64)
    z = _ih_sum(n, _stream_keys(seed, tag))
    return z.astype(np.float32) * _scale_const(std)


def _tail_exponent_np(seed: int, tag: int, start: int, count: int):
    n = np.arange(start, start + count, dtype=np.int64)
    u = _mix32(_mix32((n & M32) ^ _stream_keys(seed, tag)[0]) ^ (n >> 32)) & 0xFFFFFF
    k = np.zeros(count, dtype=np.int64)
    for j in range(1, 9):
        k = k + (u < (1 << (24 - 3 * j)))
    return k


def heavy_tail_f32_np(seed: int, tag: int, start: int, count: int) -> np.ndarray:
    """Heavy-tailed values: z * 2^k with z ~ N(0, 1) and P(k >= j) = 8^-j (k <= 8).
    The tail falls like |x|^-3, as for a Student-t with 3 degrees of freedom.
    Multiplying by a power of two is exact."""
    z = normal_f32_np(seed, tag * 2, start, count, 1.0)
    k = _tail_exponent_np(seed, tag * 2 + 1, start, count)
    return z * np.exp2(k).astype(np.float32)


# --------------------------------------------------------------------------
# torch generators (any device); identical bits to the numpy ones
# --------------------------------------------------------------------------

def normal_f32_torch(seed: int, tag: int, start: int, count: int, std: float, device):
    import torch
    n = torch.arange(start, start + count, dtype=torch.int64, device=device)
    z = _ih_sum(n, _stream_keys(seed, tag))
    return z.to(torch.float32) * torch.tensor(float(_scale_const(std)), dtype=torch.float32,
                                              device=device)


def heavy_tail_f32_torch(seed: int, tag: int, start: int, count: int, device):
    import torch
    z = normal_f32_torch(seed, tag * 2, start, count, 1.0, device)
    n = torch.arange(start, start + count, dtype=torch.int64, device=device)
    u = _mix32(_mix32((n & M32) ^ _stream_keys(seed, tag * 2 + 1)[0]) ^ (n >> 32)) & 0xFFFFFF
    k = torch.zeros(count, dtype=torch.int64, device=device)
    for j in range(1, 9):
        k = k + (u < (1 << (24 - 3 * j))).to(torch.int64)
    return z * torch.exp2(k.to(torch.float32))


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class MoEShape:
    T: int
    d: int
    f: int
    E: int
    k: int


# Sizes of the workloads (the pages give 384 experts, top-8 and 48 layers; the
# hidden sizes are assumed and stated).
SHAPES = {
    "single_gemm": None,  # A [128 x 256], W [256 x 256]
    "small_moe": MoEShape(T=2048, d=1024, f=512, E=32, k=4),
    # profiling case: full hidden sizes, 64 experts (1.1 GB of NVFP4 weights)
    "mid_moe": MoEShape(T=4096, d=4096, f=2560, E=64, k=8),
    "full_moe": MoEShape(T=16384, d=4096, f=2560, E=384, k=8),
}

# stream tags
TAG_X, TAG_W1, TAG_W2, TAG_LOGITS, TAG_DY, TAG_ACT, TAG_PAYLOAD, TAG_A, TAG_W = range(9)


def outlier_channels(seed: int, cols: int, n: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(cols, size=n, replace=False)).astype(np.int64)


def with_outliers_np(x2d: np.ndarray, chans: np.ndarray, factor: float) -> np.ndarray:
    x2d = x2d.copy()
    x2d[:, chans] = x2d[:, chans] * np.float32(factor)
    return x2d


def rows_np(seed: int, tag: int, row0: int, nrows: int, cols: int, std: float) -> np.ndarray:
    """bf16 bits of rows [row0, row0 + nrows) of a [* x cols] N(0, std) tensor."""
    return f32_to_bf16_bits(
        normal_f32_np(seed, tag, row0 * cols, nrows * cols, std).reshape(nrows, cols))


def rows_torch(seed: int, tag: int, row0: int, nrows: int, cols: int, std: float, device):
    import torch
    v = normal_f32_torch(seed, tag, row0 * cols, nrows * cols, std, device)
    return v.to(torch.bfloat16).reshape(nrows, cols)


def expert_weight_np(seed: int, tag: int, e: int, rows: int, cols: int, std: float = 0.02):
    """bf16 bits of expert e's [rows x cols] weight matrix."""
    return f32_to_bf16_bits(
        normal_f32_np(seed, tag, e * rows * cols, rows * cols, std).reshape(rows, cols))


def expert_weight_torch(seed: int, tag: int, e: int, rows: int, cols: int, device,
                        std: float = 0.02):
    import torch
    v = normal_f32_torch(seed, tag, e * rows * cols, rows * cols, std, device)
    return v.to(torch.bfloat16).reshape(rows, cols)


def logits_uniform_np(seed: int, T: int, E: int) -> np.ndarray:
    """Router logits ~ N(0, 1) i.i.d. (near-uniform expert loads), fp32."""
    return normal_f32_np(seed, TAG_LOGITS, 0, T * E, 1.0).reshape(T, E)


def logits_zipf_np(seed: int, T: int, E: int, s: float = 1.1) -> np.ndarray:
    """Router logits ln p_e + Gumbel(0, 1) with p_e proportional to rank^-s over a
    seeded random ranking of the experts: top-k of these samples k experts
    without replacement with probability proportional to p (Gumbel-top-k)."""
    rng = np.random.default_rng(seed)
    rank = rng.permutation(E) + 1
    logp = -s * np.log(rank.astype(np.float64))
    logp -= np.log(np.exp(logp).sum())
    g = rng.gumbel(size=(T, E))
    return (logp[None, :] + g).astype(np.float32)


def payload_rows_np(seed: int, row0: int, nrows: int, cols: int, chans: np.ndarray,
                    factor: float = 50.0) -> np.ndarray:
    """bf16 bits of heavy-tailed combine-payload rows with outlier channels."""
    v = heavy_tail_f32_np(seed, TAG_PAYLOAD, row0 * cols, nrows * cols).reshape(nrows, cols)
    return f32_to_bf16_bits(with_outliers_np(v, chans, factor))


def payload_rows_torch(seed: int, row0: int, nrows: int, cols: int, chans, device,
                       factor: float = 50.0):
    import torch
    v = heavy_tail_f32_torch(seed, TAG_PAYLOAD, row0 * cols, nrows * cols, device)
    v = v.reshape(nrows, cols)
    ch = torch.as_tensor(np.asarray(chans), device=device)
    v[:, ch] = v[:, ch] * torch.tensor(float(np.float32(factor)), dtype=torch.float32,
                                       device=device)
    return v.to(torch.bfloat16)


def grad_rows_np(seed: int, row0: int, nrows: int, cols: int, chans: np.ndarray,
                 std: float = 1e-3, factor: float = 100.0) -> np.ndarray:
    """bf16 bits of output-gradient rows ~ N(0, std) with outlier channels."""
    v = normal_f32_np(seed, TAG_DY, row0 * cols, nrows * cols, std).reshape(nrows, cols)
    return f32_to_bf16_bits(with_outliers_np(v, chans, factor))


def grad_rows_torch(seed: int, row0: int, nrows: int, cols: int, chans, device,
                    std: float = 1e-3, factor: float = 100.0):
    import torch
    v = normal_f32_torch(seed, TAG_DY, row0 * cols, nrows * cols, std, device).reshape(nrows, cols)
    ch = torch.as_tensor(np.asarray(chans), device=device)
    v[:, ch] = v[:, ch] * torch.tensor(float(np.float32(factor)), dtype=torch.float32,
                                       device=device)
    return v.to(torch.bfloat16)
