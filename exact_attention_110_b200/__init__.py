"""Exact softmax attention on NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libfa.so`` (declared in ``include/fa.h``). Every
step of the computation runs in the library's CUDA kernels; this module only checks and
marshals torch tensors (device memory and the current stream) into pointers and sizes. If
the library is missing, every call raises -- there is no fallback implementation.

    o, lse = forward(q, k, v, causal=False, block_mask=None, scale=None)
    dq, dk, dv = backward(q, k, v, o, do, lse, causal=False, block_mask=None, scale=None)
    o, lse = forward_decode(q, k, v, causal=False, scale=None, num_splits=0)   # Nq != Nk
    dq, dk, dv = backward_qk(q, k, v, o, do, lse, causal=False, scale=None)     # its gradients

q, k, v, o, do: bf16 (or fp16) CUDA tensors [B, H, N, d] of one type, contiguous, d in {64, 128, 256},
any N >= 1.
lse: fp32 [B, H, N]. block_mask: uint8 CUDA tensor [nb, nb] shared by every head, or one mask per
head [B, H, nb, nb] (nb = ceil(N/128)), or None.
"""
from __future__ import annotations

import ctypes
import math
from pathlib import Path

import torch

__all__ = [
    "FAError", "forward", "forward_decode", "backward", "backward_qk", "bwd_workspace_bytes", "bwd_preprocess", "bwd_main",
    "bwd_dq_finish", "last_device_status", "selftest_wait_timeout", "library", "LIB_PATH",
]

LIB_PATH = Path(__file__).resolve().with_name("libfa.so")

FA_OK, FA_ERR_INVALID, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT, FA_ERR_WORKSPACE = range(6)
FA_DTYPE_BF16, FA_DTYPE_F16 = 0, 1

_lib = None


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = library().fa_status_string(status).decode()
        super().__init__(f"{what}: {msg} (status {status})")


def library() -> ctypes.CDLL:
    """Loads libfa.so (built in-tree by ``python -m exact_attention_110_b200.build``)."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m exact_attention_110_b200.build` "
                "(there is no fallback implementation)")
        lib = ctypes.CDLL(str(LIB_PATH))
        vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        lib.fa_status_string.restype = ctypes.c_char_p
        lib.fa_status_string.argtypes = [i32]
        lib.fa_fwd.restype = i32
        lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, i32, vp, vp]
        lib.fa_bwd_workspace_bytes.restype = sz
        lib.fa_bwd_workspace_bytes.argtypes = [i32, i32, i32, i32]
        lib.fa_bwd.restype = i32
        lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, i32, vp, vp, sz, vp]
        lib.fa_bwd_preprocess.restype = i32
        lib.fa_bwd_preprocess.argtypes = [vp, vp, vp, i32, i32, i32, i32, f32, vp, sz, vp]
        lib.fa_bwd_main.restype = i32
        lib.fa_bwd_main.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, i32, vp, vp, sz, vp]
        lib.fa_bwd_dq_finish.restype = i32
        lib.fa_bwd_dq_finish.argtypes = [vp, i32, i32, i32, i32, vp, sz, vp]
        i64 = ctypes.c_longlong
        lib.fa_fwd_ex.restype = i32
        lib.fa_fwd_ex.argtypes = [i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, i32, vp, i64, vp]
        lib.fa_bwd_ex.restype = i32
        lib.fa_bwd_ex.argtypes = [i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, i32, vp, i64,
                                  vp, sz, vp]
        lib.fa_bwd_preprocess_ex.restype = i32
        lib.fa_bwd_preprocess_ex.argtypes = [i32] + list(lib.fa_bwd_preprocess.argtypes)
        lib.fa_bwd_main_ex.restype = i32
        lib.fa_bwd_main_ex.argtypes = [i32, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, i32, vp, i64, vp, sz, vp]
        lib.fa_bwd_dq_finish_ex.restype = i32
        lib.fa_bwd_dq_finish_ex.argtypes = [i32] + list(lib.fa_bwd_dq_finish.argtypes)
        lib.fa_fwd_decode_workspace_bytes.restype = sz
        lib.fa_fwd_decode_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32]
        lib.fa_fwd_decode.restype = i32
        lib.fa_fwd_decode.argtypes = [i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, i32, i32, vp, sz, vp]
        lib.fa_bwd_qk.restype = i32
        lib.fa_bwd_qk.argtypes = [i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, i32, vp, sz,
                                  vp]
        lib.fa_last_device_status.restype = i32
        lib.fa_last_device_status.argtypes = [vp]
        lib.fa_selftest_ex2.restype = i32
        lib.fa_selftest_ex2.argtypes = [vp, vp, vp, i32, vp]
        lib.fa_selftest_wait_timeout.restype = i32
        lib.fa_selftest_wait_timeout.argtypes = [ctypes.c_uint, vp]
        _lib = lib
    return _lib


def _check(status: int, what: str) -> None:
    if status != FA_OK:
        raise FAError(status, what)


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


_DTYPES = {torch.bfloat16: FA_DTYPE_BF16, torch.float16: FA_DTYPE_F16}


def _check_qkv(*ts):
    q = ts[0]
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    if q.dtype not in _DTYPES:
        raise ValueError("q, k, v (o, do) must be bf16 or fp16")
    for t in ts:
        if not t.is_cuda or t.dtype != q.dtype or not t.is_contiguous() or t.shape != q.shape:
            raise ValueError("q, k, v (o, do) must be contiguous CUDA tensors of one shape and type")
        if t.device != q.device:
            raise ValueError("all tensors must be on one device")
    return q.shape


def _check_mask(block_mask, B, H, N, dev):
    """Returns (mask, per-head stride in elements): 0 for one shared [nb, nb] mask."""
    if block_mask is None:
        return None, 0
    nb = (N + 127) // 128
    shape = tuple(block_mask.shape)
    if shape == (nb, nb):
        stride = 0
    elif shape in ((B, H, nb, nb), (B * H, nb, nb)):
        stride = nb * nb
    else:
        raise ValueError(f"block_mask must have shape ({nb}, {nb}) or ({B}, {H}, {nb}, {nb})")
    if not block_mask.is_cuda or block_mask.dtype != torch.uint8 or not block_mask.is_contiguous() \
            or block_mask.device != dev:
        raise ValueError("block_mask must be a contiguous uint8 CUDA tensor on the tensors' device")
    return block_mask, stride


def _scale(scale, d):
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def forward(q, k, v, causal: bool = False, block_mask=None, scale=None, out=None, lse=None):
    """O = softmax(scale * Q K^T [masked]) V and the per-row log-sum-exp (natural log)."""
    B, H, N, d = _check_qkv(q, k, v)
    mask, mstride = _check_mask(block_mask, B, H, N, q.device)
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), device=q.device, dtype=torch.float32) if lse is None else lse
    _check(library().fa_fwd_ex(_DTYPES[q.dtype], _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(l), B, H, N, d,
                               _scale(scale, d), int(bool(causal)), _ptr(mask), mstride, _stream(q.device)), "fa_fwd")
    return o, l


def forward_decode(q, k, v, causal: bool = False, scale=None, num_splits: int = 0, out=None, lse=None,
                   workspace=None):
    """Nq queries against Nk keys per head (q [B, H, Nq, d]; k, v [B, H, Nk, d]), the key range
    split over num_splits thread blocks (0: chosen by the library) and merged by LSE. causal
    uses the bottom-right alignment (key j visible to query i iff j <= i + Nk - Nq)."""
    if q.dim() != 4 or k.dim() != 4 or k.shape != v.shape:
        raise ValueError("q: [B, H, Nq, d]; k, v: [B, H, Nk, d]")
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if k.shape[:2] != (B, H) or k.shape[3] != d:
        raise ValueError("k and v must share q's B, H and d")
    for t in (q, k, v):
        if not t.is_cuda or t.dtype != q.dtype or not t.is_contiguous() or t.device != q.device:
            raise ValueError("q, k, v must be contiguous CUDA tensors of one type and device")
    if q.dtype not in _DTYPES:
        raise ValueError("q, k, v must be bf16 or fp16")
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, Nq), device=q.device, dtype=torch.float32) if lse is None else lse
    lib = library()
    need = int(lib.fa_fwd_decode_workspace_bytes(B, H, Nq, Nk, d, int(num_splits)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.fa_fwd_decode(_DTYPES[q.dtype], _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(l), B, H, Nq, Nk, d,
                             _scale(scale, d), int(bool(causal)), int(num_splits), _ptr(workspace), nbytes,
                             _stream(q.device)), "fa_fwd_decode")
    return o, l


def bwd_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(library().fa_bwd_workspace_bytes(B, H, N, d))


def _workspace(B, H, N, d, dev, workspace):
    need = bwd_workspace_bytes(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    return workspace, workspace.numel() * workspace.element_size()


def backward(q, k, v, o, do, lse, causal: bool = False, block_mask=None, scale=None, workspace=None,
             dq=None, dk=None, dv=None):
    """dQ, dK, dV of sum(O * dO) by recomputation from the saved LSE."""
    B, H, N, d = _check_qkv(q, k, v, o, do)
    mask, mstride = _check_mask(block_mask, B, H, N, q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    ws, nbytes = _workspace(B, H, N, d, q.device, workspace)
    _check(library().fa_bwd_ex(_DTYPES[q.dtype], _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                               _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, _scale(scale, d), int(bool(causal)),
                               _ptr(mask), mstride, _ptr(ws), nbytes, _stream(q.device)), "fa_bwd")
    return dq, dk, dv


def backward_qk(q, k, v, o, do, lse, causal: bool = False, scale=None, workspace=None, dq=None, dk=None, dv=None):
    """Gradients of forward_decode's result: q, o, do [B, H, Nq, d]; k, v [B, H, Nk, d];
    lse [B, H, Nq]. causal uses the bottom-right alignment. Returns (dq, dk, dv)."""
    if q.dim() != 4 or k.dim() != 4 or k.shape != v.shape:
        raise ValueError("q: [B, H, Nq, d]; k, v: [B, H, Nk, d]")
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if k.shape[:2] != (B, H) or k.shape[3] != d or o.shape != q.shape or do.shape != q.shape:
        raise ValueError("k, v share q's B, H and d; o and do have q's shape")
    for t in (q, k, v, o, do):
        if not t.is_cuda or t.dtype != q.dtype or not t.is_contiguous() or t.device != q.device:
            raise ValueError("q, k, v, o, do must be contiguous CUDA tensors of one type and device")
    if q.dtype not in _DTYPES:
        raise ValueError("q, k, v must be bf16 or fp16")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ws, nbytes = _workspace(B, H, Nq, d, q.device, workspace)
    _check(library().fa_bwd_qk(_DTYPES[q.dtype], _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                               _ptr(dq), _ptr(dk), _ptr(dv), B, H, Nq, Nk, d, _scale(scale, d), int(bool(causal)),
                               _ptr(ws), nbytes, _stream(q.device)), "fa_bwd_qk")
    return dq, dk, dv


def bwd_preprocess(o, do, lse, scale=None, workspace=None):
    B, H, N, d = _check_qkv(o, do)
    ws, nbytes = _workspace(B, H, N, d, o.device, workspace)
    _check(library().fa_bwd_preprocess_ex(_DTYPES[o.dtype], _ptr(o), _ptr(do), _ptr(lse), B, H, N, d,
                                          _scale(scale, d), _ptr(ws), nbytes, _stream(o.device)),
           "fa_bwd_preprocess")
    return ws


def bwd_main(q, k, v, do, workspace, causal=False, block_mask=None, scale=None, dk=None, dv=None):
    B, H, N, d = _check_qkv(q, k, v, do)
    mask, mstride = _check_mask(block_mask, B, H, N, q.device)
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    nbytes = workspace.numel() * workspace.element_size()
    _check(library().fa_bwd_main_ex(_DTYPES[q.dtype], _ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dk), _ptr(dv),
                                    B, H, N, d, _scale(scale, d), int(bool(causal)), _ptr(mask), mstride,
                                    _ptr(workspace), nbytes, _stream(q.device)), "fa_bwd_main")
    return dk, dv


def bwd_dq_finish(workspace, shape, device, dq=None, dtype=torch.bfloat16):
    B, H, N, d = shape
    dq = torch.empty(shape, dtype=dtype, device=device) if dq is None else dq
    if dq.dtype not in _DTYPES:
        raise ValueError("dq must be bf16 or fp16")
    nbytes = workspace.numel() * workspace.element_size()
    _check(library().fa_bwd_dq_finish_ex(_DTYPES[dq.dtype], _ptr(dq), B, H, N, d, _ptr(workspace), nbytes,
                                         _stream(device)), "fa_bwd_dq_finish")
    return dq


def selftest_wait_timeout(limit_us: int = 20000, device=None) -> None:
    """Enqueues the failure-detection self-test (a bounded wait that is meant to give up)."""
    dev = torch.device("cuda") if device is None else device
    _check(library().fa_selftest_wait_timeout(int(limit_us), _stream(dev)), "fa_selftest_wait_timeout")


def selftest_ex2(x):
    """The library's FMA-pipe exp2 and the special-function unit's ex2.approx on fp32 CUDA
    tensor x: returns (poly, sfu)."""
    if not x.is_cuda or x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous fp32 CUDA tensor")
    poly, sfu = torch.empty_like(x), torch.empty_like(x)
    _check(library().fa_selftest_ex2(_ptr(x), _ptr(poly), _ptr(sfu), x.numel(), _stream(x.device)),
           "fa_selftest_ex2")
    return poly, sfu


def last_device_status(device=None) -> int:
    """Synchronises the current stream and returns (and clears) the device status word."""
    dev = torch.device("cuda") if device is None else device
    return int(library().fa_last_device_status(_stream(dev)))
