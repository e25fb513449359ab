"""Shared helpers for the parity tests: seeded inputs as torch bf16 + fp64 numpy, and the
parity bars (absolute/mean error on O, absolute on LSE, relative Frobenius on gradients)."""
from __future__ import annotations

import functools

import numpy as np
import torch

import synth

# Parity bars for bf16 (and fp16) inputs drawn from N(0, 1).
O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3
GRAD_REL_FRO = 2e-2


@functools.lru_cache(maxsize=8)
def _stream(seed: int, n: int, dtype: str) -> np.ndarray:
    return synth.normal_bits(seed, n, dtype)


def make_case(B, H, N, d, seed=synth.BASE_SEED, device="cuda", with_do=True, dtype="bf16"):
    """Same bytes as synth.attention_inputs (cached: many cases share stream lengths): the
    16-bit tensors for the GPU and their exact fp64 values for the oracle."""
    n, shape = B * H * N * d, (B, H, N, d)
    names = ("q", "k", "v", "do") if with_do else ("q", "k", "v")
    offs = (synth.SEED_Q, synth.SEED_K, synth.SEED_V, synth.SEED_DO)
    bits = {k: _stream(seed + o, n, dtype).reshape(shape) for k, o in zip(names, offs)}
    gpu = {k: synth.to_torch(v, dtype, device) for k, v in bits.items()}
    f64 = {k: synth.bits_to_f32(v, dtype).astype(np.float64) for k, v in bits.items()}
    return gpu, f64


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_fwd_close(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    err = np.abs(o_gpu - o_ref)
    assert err.max() <= O_MAX_ABS, f"{what} O max|err| {err.max():.3e}"
    assert err.mean() <= O_MEAN_ABS, f"{what} O mean|err| {err.mean():.3e}"
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse_gpu), fin), f"{what} LSE finiteness differs"
    if fin.any():
        lerr = np.abs(lse_gpu[fin] - lse_ref[fin]).max()
        assert lerr <= LSE_MAX_ABS, f"{what} LSE max|err| {lerr:.3e}"


def rel_fro(a, b):
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


def assert_grads_close(gpu, ref, what=""):
    for name, a, b in zip(("dQ", "dK", "dV"), gpu, ref):
        assert np.all(np.isfinite(a)), f"{what} {name} has non-finite values"
        e = rel_fro(a, b)
        assert e <= GRAD_REL_FRO, f"{what} {name} relative Frobenius error {e:.3e}"
