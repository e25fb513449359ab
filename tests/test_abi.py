"""The C-ABI library loads without a GPU, exports every entry point include/fa.h declares,
and rejects bad arguments on the host before touching CUDA."""
import ctypes
import math
import re
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent
HEADER = ROOT / "include" / "fa.h"


@pytest.fixture(scope="module")
def lib():
    from exact_attention_110_b200 import build
    build.build()
    import exact_attention_110_b200 as fa
    return fa.library()


def declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert {"fa_fwd", "fa_bwd", "fa_bwd_workspace_bytes", "fa_last_device_status", "fa_status_string"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"libfa.so does not export {n}"


def test_status_strings(lib):
    for s in range(6):
        assert lib.fa_status_string(s).decode().startswith("FA_")
    assert lib.fa_status_string(99) == b"unknown fa_status"


FAKE = 0x10000  # 16-byte-aligned fake device address: argument checks must reject before use


def fwd(lib, q=FAKE, B=1, H=1, N=128, d=64, scale=0.125, lse=FAKE):
    return lib.fa_fwd(q, FAKE, FAKE, FAKE, lse, B, H, N, d, scale, 0, None, None)


def test_fwd_argument_checks(lib):
    assert fwd(lib, q=None) == 1                 # null pointer -> INVALID
    assert fwd(lib, q=FAKE + 2) == 1             # misaligned -> INVALID
    assert fwd(lib, lse=FAKE + 4) == 1
    assert fwd(lib, B=0) == 1 and fwd(lib, H=-1) == 1 and fwd(lib, N=0) == 1
    assert fwd(lib, scale=math.nan) == 1 and fwd(lib, scale=math.inf) == 1
    assert fwd(lib, d=96) == 2                   # unsupported head dim
    assert fwd(lib, d=512) == 2                  # (d = 256 is supported)
    assert lib.fa_bwd_workspace_bytes(1, 1, 128, 256) == 2 * 512 + 128 * 256 * 4 + 256  # and a backward one
    assert fwd(lib, N=0) == 1                    # empty sequence -> INVALID
    assert fwd(lib, B=65536, H=65536) == 2      # B*H above the TMA head coordinate's range


def test_workspace_size_and_checks(lib):
    # D, scaled LSE (fp32 each) and the fp32 dQ accumulator, each 256-byte aligned, then 256
    # bytes of work-scheduling counters.
    B, H, N, d = 2, 3, 256, 64
    vec = (B * H * N * 4 + 255) // 256 * 256
    acc = (B * H * N * d * 4 + 255) // 256 * 256
    assert lib.fa_bwd_workspace_bytes(B, H, N, d) == 2 * vec + acc + 256
    # any N: the vectors and the accumulator are padded to whole 128-row tiles
    assert lib.fa_bwd_workspace_bytes(1, 1, 100, 64) == 2 * 512 + 128 * 64 * 4 + 256
    assert lib.fa_bwd_workspace_bytes(1, 1, 0, 64) == 0
    assert lib.fa_bwd_workspace_bytes(1, 1, 128, 80) == 0
    need = lib.fa_bwd_workspace_bytes(1, 1, 128, 64)
    st = lib.fa_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0.125, 0, None,
                    FAKE, need - 1, None)
    assert st == 5                               # workspace too small
    st = lib.fa_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0.125, 0, None,
                    None, need, None)
    assert st == 5                               # workspace missing
    st = lib.fa_bwd(FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0.125, 0, None,
                    FAKE, need, None)
    assert st == 1
    assert lib.fa_bwd_dq_finish(FAKE + 8, 1, 1, 128, 64, FAKE, need, None) == 1
    assert lib.fa_bwd_main(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 48, 0.1, 0, None, FAKE, need, None) == 2


def test_ex_entry_points_check_dtype_and_mask_stride(lib):
    # the element type must be FA_DTYPE_BF16 (0) or FA_DTYPE_F16 (1); checked before anything else
    need = lib.fa_bwd_workspace_bytes(1, 1, 128, 64)
    for bad in (-1, 2, 7):
        assert lib.fa_fwd_ex(bad, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0.125, 0, None, 0, None) == 1
        assert lib.fa_bwd_ex(bad, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0.125, 0,
                             None, 0, FAKE, need, None) == 1
        assert lib.fa_bwd_dq_finish_ex(bad, FAKE, 1, 1, 128, 64, FAKE, need, None) == 1
    # valid types still get the ordinary argument checks
    for dt in (0, 1):
        assert lib.fa_fwd_ex(dt, None, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0.125, 0, None, 0, None) == 1
        assert lib.fa_fwd_ex(dt, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 96, 0.125, 0, None, 0, None) == 2
    # a per-head mask stride shorter than one ceil(N/128)^2 mask (here 3 x 3) is rejected
    for stride in (1, 8, -9):
        assert lib.fa_fwd_ex(0, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 300, 64, 0.125, 0, FAKE, stride, None) == 1
        assert lib.fa_bwd_main_ex(0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 300, 64, 0.125, 0, FAKE, stride,
                                  FAKE, lib.fa_bwd_workspace_bytes(1, 2, 300, 64), None) == 1


@pytest.mark.parametrize("scale", [0.0, -0.125])
def test_backward_needs_positive_scale(lib, scale):
    # The backward folds log2(scale) into the recomputed probabilities: scale <= 0 is refused
    # up front (the forward too: see test_forward_refuses_non_positive_scale).
    need = lib.fa_bwd_workspace_bytes(1, 1, 128, 64)
    assert lib.fa_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, scale, 0, None,
                      FAKE, need, None) == 2
    assert lib.fa_bwd_preprocess(FAKE, FAKE, FAKE, 1, 1, 128, 64, scale, FAKE, need, None) == 2
    assert lib.fa_bwd_main(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, scale, 0, None, FAKE, need, None) == 2


@pytest.mark.parametrize("scale", [0.0, -0.125, -1.0])
def test_forward_refuses_non_positive_scale(lib, scale):
    # The forward's reference max is the largest raw score times the scale (a row max of the
    # scaled scores only for scale > 0), and masked scores are -inf before scaling (NaN at
    # scale 0). Refused before any pointer is used.
    assert lib.fa_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, scale, 0, None, None) == 2
    assert lib.fa_fwd_ex(1, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, scale, 1, None, 0, None) == 2
    assert lib.fa_fwd_decode(0, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 4, 256, 64, scale, 0, 1, None, 0, None) == 2


def test_python_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import exact_attention_110_b200 as fa
    monkeypatch.setattr(fa, "LIB_PATH", tmp_path / "missing.so")
    monkeypatch.setattr(fa, "_lib", None)
    with pytest.raises(RuntimeError, match="no fallback"):
        fa.library()


def test_ex2_selftest_checks_arguments(lib):
    assert lib.fa_selftest_ex2(None, None, None, -1, None) == 1
    assert lib.fa_selftest_ex2(None, None, None, 4, None) == 1
    assert lib.fa_selftest_ex2(None, None, None, 0, None) == 0


def test_selftest_rejects_out_of_range_limit(lib):
    lib.fa_selftest_wait_timeout.restype = ctypes.c_int
    lib.fa_selftest_wait_timeout.argtypes = [ctypes.c_uint, ctypes.c_void_p]
    assert lib.fa_selftest_wait_timeout(0, None) == 1
    assert lib.fa_selftest_wait_timeout(2000000, None) == 1


def test_decode_argument_checks_and_workspace(lib):
    lib.fa_fwd_decode_workspace_bytes.restype = ctypes.c_size_t
    ws = lib.fa_fwd_decode_workspace_bytes
    # one piece: written directly, no workspace; k pieces: fp32 O / l and LSE per piece,
    # rows padded to whole 128-row tiles, each 256-byte aligned
    assert ws(1, 1, 5, 100, 64, 1) == 0
    B, H, nq, nk, d, ns = 2, 3, 5, 1000, 64, 4
    o_bytes = (B * H * ns * 128 * d * 4 + 255) // 256 * 256
    l_bytes = (B * H * ns * 128 * 4 + 255) // 256 * 256
    assert ws(B, H, nq, nk, d, ns) == o_bytes + l_bytes
    assert ws(1, 1, 5, 300, 64, 99) == ws(1, 1, 5, 300, 64, 3)  # capped at ceil(Nk / 128) pieces
    assert ws(1, 1, 0, 100, 64, 1) == 0 and ws(1, 1, 5, 100, 80, 1) == 0 and ws(1, 1, 5, 100, 64, -1) == 0
    call = lambda **kw: lib.fa_fwd_decode(kw.get("dt", 0), FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, kw.get("nq", 4),
                                          kw.get("nk", 256), kw.get("d", 64), 0.125, 0, kw.get("ns", 2), FAKE,
                                          kw.get("wsb", 1 << 30), None)
    assert call(nq=0) == 1 and call(nk=0) == 1 and call(ns=-1) == 1 and call(dt=5) == 1
    assert call(d=96) == 2
    assert call(wsb=10) == 5  # two pieces need a workspace


def test_decode_piece_choice(lib):
    """The library's piece count (num_splits = 0): enough (b, h, CTA) units for about three
    quarters of a 148-SM wave, at least two 128-key tiles per piece. A CTA holds one query tile
    when there is only one (N_q <= 128), when d = 256, or when there are at most eight
    (N_q <= 1024: two such CTAs share an SM), else two. (Without a GPU the SM count falls back to
    148, the B200's.)"""
    lib.fa_fwd_decode_workspace_bytes.restype = ctypes.c_size_t
    ws = lib.fa_fwd_decode_workspace_bytes

    def pieces(B, H, nq, nk, d):
        n0 = ws(B, H, nq, nk, d, 0)
        if n0 == 0:
            return 1
        hits = [k for k in range(2, 257) if ws(B, H, nq, nk, d, k) == n0]
        assert len(hits) == 1
        return hits[0]

    target = 3 * 148 // 4  # 111
    assert pieces(8, 16, 1, 16384, 128) == 1                    # 128 CTAs already
    assert pieces(4, 16, 1, 16384, 128) == -(-target // 64)     # 64 heads: 2 pieces
    assert pieces(1, 1, 1, 16384, 128) == 64                    # 111 wanted, capped at 128 key tiles / 2
    assert pieces(1, 1, 1, 65536, 128) == target                # 512 key tiles: 111 pieces
    assert pieces(1, 1, 1, 1024, 128) == 4                      # capped: 8 key tiles / 2
    # N_q = 200 is two query tiles, one per CTA: 128 CTAs already
    assert pieces(4, 16, 200, 16384, 128) == 1
    assert pieces(4, 16, 200, 16384, 256) == 1
    # N_q = 2000 is 16 query tiles, two per CTA: 8 CTAs per head, 32 for 4 heads
    assert pieces(1, 4, 2000, 16384, 128) == -(-target // 32)


def test_backward_checks_every_stage_before_launching(lib):
    # A misaligned dq (needed only by the last stage) must be refused before the first stage is
    # enqueued: no CUDA call is made, so this runs without a GPU.
    need = lib.fa_bwd_workspace_bytes(1, 1, 128, 64)
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.fa_bwd_noalloc.restype = i32
    lib.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, i32, vp, vp]
    args = [FAKE] * 9
    for i in range(9):
        bad = list(args)
        bad[i] = FAKE + 8
        st = lib.fa_bwd(*bad, 1, 1, 128, 64, 0.125, 0, None, FAKE, need, None)
        assert st == 1, (i, st)
        st = lib.fa_bwd_noalloc(*bad, 1, 1, 128, 64, 0.125, 0, None, None)
        assert st == 1, (i, st)
        bad[i] = None
        assert lib.fa_bwd(*bad, 1, 1, 128, 64, 0.125, 0, None, FAKE, need, None) == 1


def test_general_shape_backward_argument_checks(lib):
    i32 = ctypes.c_int
    f = lib.fa_bwd_qk
    f.restype = i32
    need = lib.fa_bwd_workspace_bytes(1, 1, 100, 64)

    def call(Nq=100, Nk=300, d=64, scale=0.125, ws=FAKE, nbytes=need, dq=FAKE, dtype=0):
        return f(dtype, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, dq, FAKE, FAKE, 1, 1, Nq, Nk, d,
                 ctypes.c_float(scale), 1, ws, ctypes.c_size_t(nbytes), None)
    assert call(dq=FAKE + 4) == 1
    assert call(Nq=0) == 1 and call(Nk=0) == 1
    assert call(d=96) == 2 and call(scale=-1.0) == 2 and call(scale=0.0) == 2
    assert call(nbytes=need - 1) == 5 and call(ws=None) == 5
    assert call(dtype=7) == 1
