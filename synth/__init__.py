"""Seeded synthetic inputs shared by the oracle checks, the CUDA parity tests and the benchmark.

This module holds no attention arithmetic. It only turns a seed into bytes:

* ``splitmix64(seed, n)`` -- the SplitMix64 generator of Steele, Lea and Flood
  ("Fast splittable pseudorandom number generators", OOPSLA 2014), written in its
  counter form: the i-th output (i = 0, 1, ...) is ``mix(seed + (i + 1) * gamma)``
  with gamma = 0x9E3779B97F4A7C15 and the published 64-bit finaliser ``mix``.
* ``normal_bf16(seed, n)`` -- standard normal draws by the Box-Muller transform
  (Box and Muller, 1958) on pairs of uniforms u = (x >> 11) * 2^-53, rounded
  fp64 -> fp32 -> bf16, both with round-to-nearest-even. The result is returned
  as raw bf16 bit patterns (uint16), so the GPU path and the oracle can be fed the
  very same bytes.
* ``bernoulli_block_mask(seed, nb, p)`` -- a row-major nb x nb uint8 block mask,
  entry on iff its uniform draw is below p, diagonal forced on.

Seeds follow one convention everywhere: Q = base + 0, K = base + 1, V = base + 2,
dO = base + 3, block mask = base + 4.
"""
from __future__ import annotations

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

BASE_SEED = 20261202
SEED_Q, SEED_K, SEED_V, SEED_DO, SEED_MASK = 0, 1, 2, 3, 4

# Generating very long streams in one piece would allocate several uint64 temporaries
# of the full length; chunking keeps peak host memory modest.
_CHUNK = 1 << 22


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64(seed: int, n: int, start: int = 0) -> np.ndarray:
    """Outputs start .. start+n-1 of the SplitMix64 stream seeded with ``seed``."""
    out = np.empty(n, dtype=np.uint64)
    s = np.uint64(seed & 0xFFFFFFFFFFFFFFFF)
    with np.errstate(over="ignore"):
        for lo in range(0, n, _CHUNK):
            hi = min(n, lo + _CHUNK)
            ctr = np.arange(start + lo + 1, start + hi + 1, dtype=np.uint64)
            out[lo:hi] = _mix64(s + ctr * GAMMA)
    return out


def uniform01(seed: int, n: int, start: int = 0) -> np.ndarray:
    """Uniform doubles in [0, 1): the top 53 bits of each SplitMix64 output."""
    x = splitmix64(seed, n, start)
    return (x >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); finite inputs only."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    return ((b + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to IEEE fp16 (round to nearest, ties to even) as bit patterns."""
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def f16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen fp16 bit patterns to fp32 (exact)."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float32)


def _normal_bits(seed: int, n: int, to_bits) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    npairs_total = (n + 1) // 2
    for lo in range(0, npairs_total, _CHUNK):
        hi = min(npairs_total, lo + _CHUNK)
        u = uniform01(seed, 2 * (hi - lo), start=2 * lo)
        u1, u2 = u[0::2], u[1::2]
        r = np.sqrt(-2.0 * np.log1p(-u1))  # 1 - u1 lies in (0, 1], so the log is finite
        theta = 2.0 * np.pi * u2
        z = np.empty(2 * (hi - lo), dtype=np.float64)
        z[0::2] = r * np.cos(theta)
        z[1::2] = r * np.sin(theta)
        m = min(n - 2 * lo, z.size)
        out[2 * lo:2 * lo + m] = to_bits(z[:m].astype(np.float32))
    return out


def normal_bf16(seed: int, n: int) -> np.ndarray:
    """n standard-normal draws as bf16 bit patterns (uint16)."""
    return _normal_bits(seed, n, f32_to_bf16_bits)


def normal_f16(seed: int, n: int) -> np.ndarray:
    """The same n standard-normal draws as fp16 bit patterns (uint16)."""
    return _normal_bits(seed, n, f32_to_f16_bits)


def normal_bits(seed: int, n: int, dtype: str = "bf16") -> np.ndarray:
    return normal_f16(seed, n) if dtype == "f16" else normal_bf16(seed, n)


def bits_to_f32(bits: np.ndarray, dtype: str = "bf16") -> np.ndarray:
    return f16_bits_to_f32(bits) if dtype == "f16" else bf16_bits_to_f32(bits)


def bernoulli_block_mask(seed: int, nb: int, p: float = 0.25, force_diagonal: bool = True) -> np.ndarray:
    """Row-major nb x nb uint8 block mask: 1 iff the entry's uniform draw is < p."""
    u = uniform01(seed, nb * nb).reshape(nb, nb)
    m = (u < p).astype(np.uint8)
    if force_diagonal:
        np.fill_diagonal(m, 1)
    return m


def attention_inputs(B: int, H: int, N: int, d: int, base_seed: int = BASE_SEED, with_do: bool = True,
                     dtype: str = "bf16"):
    """Q, K, V (and dO) for a [B, H, N, d] problem as bf16 (or fp16) bit arrays of that shape."""
    shape = (B, H, N, d)
    n = B * H * N * d
    out = {
        "q": normal_bits(base_seed + SEED_Q, n, dtype).reshape(shape),
        "k": normal_bits(base_seed + SEED_K, n, dtype).reshape(shape),
        "v": normal_bits(base_seed + SEED_V, n, dtype).reshape(shape),
    }
    if with_do:
        out["do"] = normal_bits(base_seed + SEED_DO, n, dtype).reshape(shape)
    return out


def block_mask_for(N: int, base_seed: int = BASE_SEED, p: float = 0.25, block: int = 128) -> np.ndarray:
    nb = (N + block - 1) // block
    return bernoulli_block_mask(base_seed + SEED_MASK, nb, p)


def to_torch_bf16(bits: np.ndarray, device="cpu"):
    """The bf16 bit patterns as a torch.bfloat16 tensor on `device` (bit-exact)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def to_torch(bits: np.ndarray, dtype: str = "bf16", device="cpu"):
    """bf16 or fp16 bit patterns as a torch tensor of that type on `device` (bit-exact)."""
    import torch

    tdt = torch.float16 if dtype == "f16" else torch.bfloat16
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(tdt)
    return t.to(device)
