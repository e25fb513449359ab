"""GPU parity: the CUDA kernels (through the C ABI) against the fp64 oracle on the same
seeded bf16 inputs, element by element, with the bars in tests/helpers.py."""
import numpy as np
import pytest
import torch

import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import exact_attention_110_b200 as fa
    fa.library()
    return fa


def run_fwd(fa, gpu, causal, mask_t, scale):
    o, lse = fa.forward(gpu["q"], gpu["k"], gpu["v"], causal=causal, block_mask=mask_t, scale=scale)
    torch.cuda.synchronize()
    assert fa.last_device_status() == 0
    return o, lse


def run_bwd(fa, gpu, o, lse, causal, mask_t, scale):
    dq, dk, dv = fa.backward(gpu["q"], gpu["k"], gpu["v"], o, gpu["do"], lse, causal=causal,
                             block_mask=mask_t, scale=scale)
    torch.cuda.synchronize()
    assert fa.last_device_status() == 0
    return dq, dk, dv


def mask_for(kind, N, seed=synth.BASE_SEED):
    nb = (N + 127) // 128
    if kind is None:
        return None
    if kind == "bernoulli":
        return synth.block_mask_for(N, seed)
    if kind == "ones":
        return np.ones((nb, nb), np.uint8)
    if kind == "diag":
        return np.eye(nb, dtype=np.uint8)
    raise ValueError(kind)


SMALL = [
    # B, H, N, d, causal, mask
    (1, 1, 128, 64, False, None),      # tiny config: one tile
    (1, 2, 384, 64, False, None),      # odd number of 128-row tiles (last CTA has one tile)
    (1, 2, 384, 128, False, None),
    (2, 1, 640, 64, True, None),
    (1, 2, 512, 128, True, None),
    (1, 2, 512, 64, False, "bernoulli"),
    (1, 1, 768, 128, True, "bernoulli"),
    (1, 1, 512, 64, False, "diag"),
    # ragged sequence lengths: a partial last tile of queries and keys
    (1, 1, 1, 64, False, None),        # a single query and key
    (1, 2, 77, 64, True, None),        # one partial tile
    (2, 1, 130, 64, False, "bernoulli"),
    (1, 2, 200, 128, False, None),
    (1, 1, 333, 128, True, None),
    (1, 1, 641, 64, True, "bernoulli"),
    (1, 1, 1000, 128, False, None),
    # a single query tile runs the one-tile kernel (S double-buffered, columns split)
    (1, 2, 100, 128, True, None),
    (2, 1, 128, 128, False, "bernoulli"),
    # at most 32 (64) rows at d = 64: four (two) copies of the rows, each scoring its share of
    # every step's keys, combined at the end; just past that, the per-row form of the same kernel
    (1, 3, 32, 64, True, None),
    (2, 1, 20, 64, False, "ones"),
    (2, 1, 33, 64, False, None),
    (1, 2, 64, 64, True, None),
    (1, 1, 65, 64, True, None),
]


@pytest.mark.parametrize("B,Hh,N,d,causal,mask", SMALL)
def test_fwd_bwd_small(fa, oracle_mod, B, Hh, N, d, causal, mask):
    gpu, ref = H.make_case(B, Hh, N, d, seed=synth.BASE_SEED + N + d)
    scale = 1.0 / np.sqrt(d)
    m = mask_for(mask, N)
    mt = None if m is None else torch.from_numpy(m).cuda()
    o, lse = run_fwd(fa, gpu, causal, mt, scale)
    o_ref, lse_ref = oracle_mod.attention_fwd(ref["q"], ref["k"], ref["v"], scale, causal=causal, mask=m)
    H.assert_fwd_close(H.to_f64(o), H.to_f64(lse), o_ref, lse_ref, f"fwd {B,Hh,N,d,causal,mask}")
    dq, dk, dv = run_bwd(fa, gpu, o, lse, causal, mt, scale)
    g_ref = oracle_mod.attention_bwd(ref["q"], ref["k"], ref["v"], ref["do"], scale, causal=causal, mask=m)[:3]
    H.assert_grads_close([H.to_f64(x) for x in (dq, dk, dv)], g_ref, f"bwd {B,Hh,N,d,causal,mask}")


FP16 = [
    # B, H, N, d, causal, mask: fp16 inputs and outputs through the *_ex entry points
    (1, 2, 384, 64, False, None),
    (2, 1, 640, 64, True, None),
    (1, 2, 512, 128, True, None),
    (1, 1, 333, 128, False, "bernoulli"),
    (1, 2, 96, 128, True, None),       # one query tile: the one-tile kernel in fp16
]


@pytest.mark.parametrize("B,Hh,N,d,causal,mask", FP16)
def test_fwd_bwd_fp16(fa, oracle_mod, B, Hh, N, d, causal, mask):
    gpu, ref = H.make_case(B, Hh, N, d, seed=synth.BASE_SEED + 3 * N + d, dtype="f16")
    assert gpu["q"].dtype == torch.float16
    scale = 1.0 / np.sqrt(d)
    m = mask_for(mask, N)
    mt = None if m is None else torch.from_numpy(m).cuda()
    o, lse = run_fwd(fa, gpu, causal, mt, scale)
    assert o.dtype == torch.float16
    o_ref, lse_ref = oracle_mod.attention_fwd(ref["q"], ref["k"], ref["v"], scale, causal=causal, mask=m)
    H.assert_fwd_close(H.to_f64(o), H.to_f64(lse), o_ref, lse_ref, f"fp16 fwd {B,Hh,N,d,causal,mask}")
    dq, dk, dv = run_bwd(fa, gpu, o, lse, causal, mt, scale)
    assert dq.dtype == dk.dtype == dv.dtype == torch.float16
    g_ref = oracle_mod.attention_bwd(ref["q"], ref["k"], ref["v"], ref["do"], scale, causal=causal, mask=m)[:3]
    H.assert_grads_close([H.to_f64(x) for x in (dq, dk, dv)], g_ref, f"fp16 bwd {B,Hh,N,d,causal,mask}")


@pytest.mark.parametrize("B,Hh,N,d,causal", [(2, 2, 640, 64, False), (1, 3, 513, 128, True)])
def test_per_head_block_masks(fa, oracle_mod, B, Hh, N, d, causal):
    # Every (b, h) has its own Bernoulli mask, of a different density; each head must match the
    # oracle run with that head's mask.
    gpu, ref = H.make_case(B, Hh, N, d, seed=synth.BASE_SEED + 17 + N)
    nb = (N + 127) // 128
    masks = np.stack([synth.bernoulli_block_mask(synth.BASE_SEED + 100 + x, nb, p=0.15 + 0.2 * x)
                      for x in range(B * Hh)]).reshape(B, Hh, nb, nb)
    scale = 1.0 / np.sqrt(d)
    mt = torch.from_numpy(masks).cuda()
    o, lse = run_fwd(fa, gpu, causal, mt, scale)
    dq, dk, dv = run_bwd(fa, gpu, o, lse, causal, mt, scale)
    outs = [H.to_f64(x) for x in (o, lse, dq, dk, dv)]
    for b in range(B):
        for h in range(Hh):
            sl = (slice(b, b + 1), slice(h, h + 1))
            args = [ref[k][sl] for k in ("q", "k", "v")]
            o_ref, l_ref = oracle_mod.attention_fwd(*args, scale, causal=causal, mask=masks[b, h])
            H.assert_fwd_close(outs[0][sl], outs[1][sl], o_ref, l_ref, f"head {b},{h}")
            g_ref = oracle_mod.attention_bwd(*args, ref["do"][sl], scale, causal=causal, mask=masks[b, h])[:3]
            H.assert_grads_close([x[sl] for x in outs[2:]], g_ref, f"head {b},{h}")


HEAD_DIM_256 = [
    # B, H, N, causal, mask, dtype: d = 256 (forward: one query tile per CTA; backward: two CTAs
    # per key tile, one per 128-column half of d, Q/dO/V streamed as 64-column panels)
    (1, 2, 384, False, None, "bf16"),
    (2, 1, 333, True, None, "bf16"),       # ragged, causal
    (1, 1, 640, False, "bernoulli", "bf16"),
    (1, 2, 128, True, None, "bf16"),       # a single tile
    (1, 1, 1000, True, None, "bf16"),      # many query tiles per key tile: the ring wraps often
    (1, 2, 520, False, None, "f16"),
]


@pytest.mark.parametrize("B,Hh,N,causal,mask,dtype", HEAD_DIM_256)
def test_head_dim_256(fa, oracle_mod, B, Hh, N, causal, mask, dtype):
    d = 256
    gpu, ref = H.make_case(B, Hh, N, d, seed=synth.BASE_SEED + N + 256, dtype=dtype)
    scale = 1.0 / np.sqrt(d)
    m = mask_for(mask, N)
    mt = None if m is None else torch.from_numpy(m).cuda()
    o, lse = run_fwd(fa, gpu, causal, mt, scale)
    o_ref, l_ref = oracle_mod.attention_fwd(ref["q"], ref["k"], ref["v"], scale, causal=causal, mask=m)
    H.assert_fwd_close(H.to_f64(o), H.to_f64(lse), o_ref, l_ref, f"d=256 fwd {B,Hh,N,causal,mask,dtype}")
    dq, dk, dv = run_bwd(fa, gpu, o, lse, causal, mt, scale)
    g_ref = oracle_mod.attention_bwd(ref["q"], ref["k"], ref["v"], ref["do"], scale, causal=causal, mask=m)[:3]
    H.assert_grads_close([H.to_f64(x) for x in (dq, dk, dv)], g_ref, f"d=256 bwd {B,Hh,N,causal,mask,dtype}")


def test_head_dim_256_sweep_shape(fa, oracle_mod):
    # The sweep's 16k-token, hidden-2048 batch at d = 256 (B = 4, H = 8, N = 4096) in one launch
    # of each kernel; one sampled head against the oracle in full.
    check_heads(fa, oracle_mod, 4, 8, 4096, 256, True, None, nheads=1, seed=synth.BASE_SEED + 256)


def test_head_dim_256_general_shape(fa, oracle_mod):
    # d = 256 through the general-shape backward (N_q != N_k, bottom-right causal)
    B, Hh, Nq, Nk, d = 1, 2, 200, 450, 256
    seed = synth.BASE_SEED + 4
    gq, rq = H.make_case(B, Hh, Nq, d, seed=seed)
    gk, rk = H.make_case(B, Hh, Nk, d, seed=seed + 500, with_do=False)
    scale = 1.0 / np.sqrt(d)
    o, lse = fa.forward_decode(gq["q"], gk["k"], gk["v"], causal=True, scale=scale)
    dq, dk, dv = fa.backward_qk(gq["q"], gk["k"], gk["v"], o, gq["do"], lse, causal=True, scale=scale)
    torch.cuda.synchronize()
    assert fa.last_device_status() == 0
    g_ref = oracle_mod.attention_bwd_qk(rq["q"], rk["k"], rk["v"], rq["do"], scale, causal=True)[:3]
    H.assert_grads_close([H.to_f64(x) for x in (dq, dk, dv)], g_ref, "d=256 general bwd")


DECODE = [
    # B, H, Nq, Nk, d, causal, num_splits (0: the library's choice), dtype
    (2, 4, 1, 4096, 128, False, 0, "bf16"),      # one query per head, long key history
    (1, 2, 16, 1000, 64, True, 0, "bf16"),       # bottom-right causal, ragged key tail
    (1, 2, 130, 777, 128, True, 3, "bf16"),      # two query tiles, uneven pieces
    (1, 1, 300, 200, 64, True, 2, "bf16"),       # more queries than keys: 100 rows see nothing
    (2, 1, 64, 2048, 128, False, 1, "bf16"),     # one piece: written directly, no merge
    (1, 3, 8, 3000, 64, False, 5, "f16"),
    (1, 2, 40, 900, 256, True, 0, "bf16"),      # head dim 256
    (2, 2, 4, 5000, 128, True, 0, "f16"),       # fp16, bottom-right causal, library's split
    (2, 3, 32, 16384, 64, False, 0, "bf16"),    # 32 queries at d = 64: four row copies, library's split
    (1, 2, 5, 3, 64, True, 0, "bf16"),          # fewer keys than queries: rows 0-1 see no key
    (3, 1, 1, 130, 64, False, 0, "bf16"),       # one query, a ragged second key tile
    (1, 2, 33, 700, 64, True, 0, "f16"),        # 33 queries: two copies of 64 rows
    (2, 2, 64, 16384, 64, True, 0, "bf16"),     # 64 queries, bottom-right causal, library's split
    (1, 3, 40, 1000, 64, False, 3, "bf16"),     # two copies, three key-range pieces
]


@pytest.mark.parametrize("B,Hh,Nq,Nk,d,causal,splits,dtype", DECODE)
def test_decode_forward(fa, oracle_mod, B, Hh, Nq, Nk, d, causal, splits, dtype):
    seed = synth.BASE_SEED + 31 * Nq + Nk
    gq, rq = H.make_case(B, Hh, Nq, d, seed=seed, with_do=False, dtype=dtype)
    gk, rk = H.make_case(B, Hh, Nk, d, seed=seed + 1000, with_do=False, dtype=dtype)
    scale = 1.0 / np.sqrt(d)
    o, lse = fa.forward_decode(gq["q"], gk["k"], gk["v"], causal=causal, scale=scale, num_splits=splits)
    torch.cuda.synchronize()
    assert fa.last_device_status() == 0
    o_ref, l_ref = oracle_mod.attention_fwd_qk(rq["q"], rk["k"], rk["v"], scale, causal=causal)
    H.assert_fwd_close(H.to_f64(o), H.to_f64(lse), o_ref, l_ref, f"decode {B,Hh,Nq,Nk,d,causal,splits}")


def test_decode_path_agrees_with_square_forward(fa):
    # Nq = Nk through the split-and-merge path gives the square forward's result up to rounding
    gpu, _ = H.make_case(1, 2, 640, 128, seed=synth.BASE_SEED + 77, with_do=False)
    for causal in (False, True):
        o1, l1 = run_fwd(fa, gpu, causal, None, 0.0884)
        o2, l2 = fa.forward_decode(gpu["q"], gpu["k"], gpu["v"], causal=causal, scale=0.0884, num_splits=3)
        torch.cuda.synchronize()
        assert (o1.float() - o2.float()).abs().max().item() < 8e-3
        assert (l1 - l2).abs().max().item() < 1e-4


def test_fp16_and_bf16_agree(fa):
    # The same draws rounded to each type give nearly the same attention: the element type
    # only changes input rounding and the 16-bit P (fp16 carries three more mantissa bits).
    g16, _ = H.make_case(1, 2, 512, 128, seed=synth.BASE_SEED + 5, dtype="f16")
    gbf, _ = H.make_case(1, 2, 512, 128, seed=synth.BASE_SEED + 5, dtype="bf16")
    o16, l16 = run_fwd(fa, g16, False, None, 0.0884)
    obf, lbf = run_fwd(fa, gbf, False, None, 0.0884)
    assert (o16.float() - obf.float()).abs().max().item() < 3e-2
    assert (l16 - lbf).abs().max().item() < 3e-2


def sampled_heads(B, Hh, n, seed):
    rng = np.random.default_rng(seed)
    flat = rng.choice(B * Hh, size=min(n, B * Hh), replace=False)
    return [(int(f // Hh), int(f % Hh)) for f in sorted(flat)]


def check_heads(fa, oracle_mod, B, Hh, N, d, causal, mask, nheads, seed):
    gpu, ref = H.make_case(B, Hh, N, d, seed=seed)
    scale = 1.0 / np.sqrt(d)
    mt = None if mask is None else torch.from_numpy(mask).cuda()
    o, lse = run_fwd(fa, gpu, causal, mt, scale)
    dq, dk, dv = run_bwd(fa, gpu, o, lse, causal, mt, scale)
    outs = [H.to_f64(x) for x in (o, lse, dq, dk, dv)]
    for (b, h) in sampled_heads(B, Hh, nheads, seed):
        sl = (slice(b, b + 1), slice(h, h + 1))
        args = [ref[k][sl] for k in ("q", "k", "v")]
        o_ref, lse_ref = oracle_mod.attention_fwd(*args, scale, causal=causal, mask=mask)
        H.assert_fwd_close(outs[0][sl], outs[1][sl], o_ref, lse_ref, f"head {b},{h}")
        g_ref = oracle_mod.attention_bwd(*args, ref["do"][sl], scale, causal=causal, mask=mask)[:3]
        H.assert_grads_close([x[sl] for x in outs[2:]], g_ref, f"head {b},{h}")


def test_config_bert_large_shape(fa, oracle_mod):
    # B=16, H=16, N=512, d=64, non-causal (sampled heads checked in full)
    check_heads(fa, oracle_mod, 16, 16, 512, 64, False, None, nheads=8, seed=synth.BASE_SEED)


def test_config_gpt2_shape_causal(fa, oracle_mod):
    # B=8, H=12, N=1024, d=64, causal
    check_heads(fa, oracle_mod, 8, 12, 1024, 64, True, None, nheads=4, seed=synth.BASE_SEED)


def test_config_block_sparse(fa, oracle_mod):
    # B=4, H=16, N=4096, d=64, 128x128 blocks: diagonal on, others Bernoulli(0.25)
    mask = synth.block_mask_for(4096, synth.BASE_SEED)
    check_heads(fa, oracle_mod, 4, 16, 4096, 64, False, mask, nheads=1, seed=synth.BASE_SEED)


@pytest.mark.parametrize("N", [512, 1024, 2048, 4096, 8192, 16384])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_config_seqlen_sweep_forward_and_backward(fa, oracle_mod, N, d, causal):
    # 16k tokens, hidden 2048: B = 16384 / N, H = 2048 / d, one launch of each kernel over the
    # whole batch as the benchmark runs it. One sampled head is compared with the oracle in
    # full: O and LSE, and dQ, dK, dV of the recomputation backward ([P3] §4.2: the same
    # gradients as the standard backward).
    B, Hh = 16384 // N, 2048 // d
    gpu, ref = H.make_case(B, Hh, N, d, seed=synth.BASE_SEED + 7)
    scale = 1.0 / np.sqrt(d)
    o, lse = run_fwd(fa, gpu, causal, None, scale)
    dq, dk, dv = run_bwd(fa, gpu, o, lse, causal, None, scale)
    for (b, h) in sampled_heads(B, Hh, 1, N + d + causal):
        sl = (slice(b, b + 1), slice(h, h + 1))
        outs = [H.to_f64(x[sl]) for x in (o, lse, dq, dk, dv)]
        args = [ref[k][sl] for k in ("q", "k", "v")]
        o_ref, l_ref = oracle_mod.attention_fwd(*args, scale, causal=causal)
        H.assert_fwd_close(outs[0], outs[1], o_ref, l_ref, f"N={N} d={d} causal={causal} head {b},{h}")
        g_ref = oracle_mod.attention_bwd(*args, ref["do"][sl], scale, causal=causal)[:3]
        H.assert_grads_close(outs[2:], g_ref, f"N={N} d={d} causal={causal} head {b},{h}")


GENERAL_BWD = [
    # B, H, Nq, Nk, d, causal, dtype: the backward of N_q queries against N_k keys
    (1, 2, 128, 512, 64, False, "bf16"),
    (1, 2, 200, 700, 128, True, "bf16"),     # ragged, bottom-right causal: rows see different key counts
    (2, 1, 300, 200, 64, True, "bf16"),      # more queries than keys: 100 rows see nothing
    (1, 1, 1, 1000, 128, True, "bf16"),      # one query (a decode step's gradient)
    (1, 2, 640, 256, 128, False, "bf16"),
    (1, 2, 384, 1000, 64, True, "f16"),
    (1, 1, 512, 512, 128, True, "bf16"),     # N_q = N_k through the general entry point
]


@pytest.mark.parametrize("B,Hh,Nq,Nk,d,causal,dtype", GENERAL_BWD)
def test_general_shape_backward(fa, oracle_mod, B, Hh, Nq, Nk, d, causal, dtype):
    seed = synth.BASE_SEED + 13 * Nq + Nk
    gq, rq = H.make_case(B, Hh, Nq, d, seed=seed, dtype=dtype)
    gk, rk = H.make_case(B, Hh, Nk, d, seed=seed + 500, with_do=False, dtype=dtype)
    scale = 1.0 / np.sqrt(d)
    o, lse = fa.forward_decode(gq["q"], gk["k"], gk["v"], causal=causal, scale=scale)
    dq, dk, dv = fa.backward_qk(gq["q"], gk["k"], gk["v"], o, gq["do"], lse, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.last_device_status() == 0
    assert dq.shape == gq["q"].shape and dk.shape == dv.shape == gk["k"].shape
    o_ref, l_ref = oracle_mod.attention_fwd_qk(rq["q"], rk["k"], rk["v"], scale, causal=causal)
    H.assert_fwd_close(H.to_f64(o), H.to_f64(lse), o_ref, l_ref, f"general fwd {B,Hh,Nq,Nk,d,causal}")
    g_ref = oracle_mod.attention_bwd_qk(rq["q"], rk["k"], rk["v"], rq["do"], scale, causal=causal)[:3]
    H.assert_grads_close([H.to_f64(x) for x in (dq, dk, dv)], g_ref, f"general bwd {B,Hh,Nq,Nk,d,causal}")
    if causal and Nq > Nk:  # rows that see no key: dQ exactly zero
        assert torch.all(dq[:, :, :Nq - Nk] == 0)


def test_general_shape_backward_equals_square_backward(fa):
    # N_q = N_k: the general entry point runs the same kernels as fa_bwd, so dK and dV are
    # bit-identical; dQ differs at most by the order in which key tiles' shares were added.
    gpu, _ = H.make_case(1, 2, 640, 128, seed=synth.BASE_SEED + 78)
    for causal in (False, True):
        o, lse = run_fwd(fa, gpu, causal, None, 0.0884)
        dq1, dk1, dv1 = run_bwd(fa, gpu, o, lse, causal, None, 0.0884)
        dq2, dk2, dv2 = fa.backward_qk(gpu["q"], gpu["k"], gpu["v"], o, gpu["do"], lse, causal=causal, scale=0.0884)
        torch.cuda.synchronize()
        assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
        assert (dq1.float() - dq2.float()).abs().max().item() < 2e-3


def test_misaligned_dq_leaves_outputs_untouched(fa):
    # Every argument of every backward stage is checked before the first launch: a bad dq
    # (used only by the last stage) must not let the first two stages write dK and dV.
    import ctypes
    gpu, _ = H.make_case(1, 1, 256, 64, seed=synth.BASE_SEED + 79)
    o, lse = run_fwd(fa, gpu, False, None, 0.125)
    dk = torch.full_like(gpu["q"], 3.0)
    dv = torch.full_like(gpu["q"], -2.0)
    dq_buf = torch.zeros(gpu["q"].numel() + 8, dtype=gpu["q"].dtype, device="cuda")
    ws = torch.empty(fa.bwd_workspace_bytes(1, 1, 256, 64), dtype=torch.uint8, device="cuda")
    lib = fa.library()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.fa_bwd(gpu["q"].data_ptr(), gpu["k"].data_ptr(), gpu["v"].data_ptr(), o.data_ptr(), gpu["do"].data_ptr(),
                    lse.data_ptr(), dq_buf.data_ptr() + 2, dk.data_ptr(), dv.data_ptr(), 1, 1, 256, 64, 0.125, 0,
                    None, ws.data_ptr(), ws.numel(), stream)
    torch.cuda.synchronize()
    assert st == 1
    assert torch.all(dk == 3.0) and torch.all(dv == -2.0)


@pytest.mark.parametrize("N,d", [(256, 64), (640, 128), (300, 256)])
def test_causal_grid_order_with_a_partial_last_group(fa, oracle_mod, N, d):
    # Causal grids enumerate heads in groups (longest work items first within a group); with
    # 300 heads the last group is partial. Heads at both ends and inside the partial group must
    # match the oracle in both passes.
    B, Hh = 100, 3
    gpu, ref = H.make_case(B, Hh, N, d, seed=synth.BASE_SEED + 300 + N)
    scale = 1.0 / np.sqrt(d)
    o, lse = run_fwd(fa, gpu, True, None, scale)
    dq, dk, dv = run_bwd(fa, gpu, o, lse, True, None, scale)
    for (b, h) in ((0, 0), (49, 1), (98, 2), (99, 0), (99, 2)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        args = [ref[k][sl] for k in ("q", "k", "v")]
        o_ref, l_ref = oracle_mod.attention_fwd(*args, scale, causal=True)
        H.assert_fwd_close(H.to_f64(o[sl]), H.to_f64(lse[sl]), o_ref, l_ref, f"head {b},{h}")
        g_ref = oracle_mod.attention_bwd(*args, ref["do"][sl], scale, causal=True)[:3]
        H.assert_grads_close([H.to_f64(x[sl]) for x in (dq, dk, dv)], g_ref, f"head {b},{h}")


def test_masked_blocks_do_not_influence_output(fa):
    # Keys/values in blocks that are off (or in the causal future) must not change O at all.
    N, d = 512, 64
    gpu, _ = H.make_case(1, 2, N, d, seed=11)
    m = np.array([[1, 0, 0, 0], [1, 1, 0, 0], [0, 1, 1, 0], [1, 0, 0, 1]], np.uint8)
    mt = torch.from_numpy(m).cuda()
    o1, l1 = run_fwd(fa, gpu, False, mt, 0.125)
    k2, v2 = gpu["k"].clone(), gpu["v"].clone()
    k2[:, :, 128:256] += 3.0   # key block 1 is visible only to query blocks 1, 2
    v2[:, :, 128:256] -= 5.0
    gpu2 = dict(gpu, k=k2, v=v2)
    o2, l2 = run_fwd(fa, gpu2, False, mt, 0.125)
    assert torch.equal(o1[:, :, :128], o2[:, :, :128]) and torch.equal(o1[:, :, 384:], o2[:, :, 384:])
    assert torch.equal(l1[:, :, :128], l2[:, :, :128])
    # causal: perturbing the last key block changes nothing for earlier query blocks
    o3, _ = run_fwd(fa, gpu, True, None, 0.125)
    k4 = gpu["k"].clone()
    k4[:, :, 384:] *= -2.0
    o4, _ = run_fwd(fa, dict(gpu, k=k4), True, None, 0.125)
    assert torch.equal(o3[:, :, :384], o4[:, :, :384])


def test_fully_masked_query_block(fa, oracle_mod):
    # Query block 0 sees no key block: O = 0, LSE = -inf, and its dQ is exactly zero.
    N, d = 384, 64
    gpu, ref = H.make_case(1, 1, N, d, seed=12)
    m = np.array([[0, 0, 0], [1, 1, 0], [0, 1, 1]], np.uint8)
    mt = torch.from_numpy(m).cuda()
    o, lse = run_fwd(fa, gpu, False, mt, 0.125)
    assert torch.all(o[:, :, :128] == 0) and torch.all(torch.isneginf(lse[:, :, :128]))
    o_ref, l_ref = oracle_mod.attention_fwd(ref["q"], ref["k"], ref["v"], 0.125, mask=m)
    H.assert_fwd_close(H.to_f64(o), H.to_f64(lse), o_ref, l_ref, "fully masked block")
    dq, dk, dv = run_bwd(fa, gpu, o, lse, False, mt, 0.125)
    assert torch.all(dq[:, :, :128] == 0)
    g_ref = oracle_mod.attention_bwd(ref["q"], ref["k"], ref["v"], ref["do"], 0.125, mask=m)[:3]
    H.assert_grads_close([H.to_f64(x) for x in (dq, dk, dv)], g_ref, "fully masked block")


def test_bounded_wait_timeout_is_reported_and_context_survives(fa):
    # A device-side wait that runs out (on a barrier nothing arrives at) must be reported as
    # FA_ERR_TIMEOUT by the host and leave the context usable for the next call.
    assert fa.last_device_status() == 0
    fa.selftest_wait_timeout(20000)
    assert fa.last_device_status() == 4  # FA_ERR_TIMEOUT, and the word is cleared
    assert fa.last_device_status() == 0
    gpu, _ = H.make_case(1, 1, 256, 64, seed=13)
    o, lse = run_fwd(fa, gpu, False, None, 0.125)
    assert torch.isfinite(o.float()).all()


@pytest.mark.parametrize("scale", [0.5, 3.0])
@pytest.mark.parametrize("causal", [False, True])
def test_large_scale_exercises_the_rescale_path(fa, oracle_mod, scale, causal):
    # With scale well above 1/sqrt(d) the row maxima jump by far more than the reference-max
    # threshold from tile to tile, so O is rescaled in TMEM over and over; P is nearly one-hot.
    # The absolute bars assume scale = 1/sqrt(d), where O averages many rows of V and stays
    # small. Here |O| approaches single rows of V (up to ~4.5), where half a bf16 ulp alone is
    # up to 2^-7 and P's own 2^-9 rounding adds as much again: the bar is relative to |O|
    # (1% of max(1, |O|)), the mean is 2e-3, and the LSE (up to ~100) is held to 1e-3 of
    # max(1, |LSE|).
    N, d = 1000, 128
    gpu, ref = H.make_case(1, 2, N, d, seed=synth.BASE_SEED + 41)
    o, lse = run_fwd(fa, gpu, causal, None, scale)
    o_ref, l_ref = oracle_mod.attention_fwd(ref["q"], ref["k"], ref["v"], scale, causal=causal)
    err = np.abs(H.to_f64(o) - o_ref)
    assert (err / np.maximum(1.0, np.abs(o_ref))).max() <= 1e-2, f"scale {scale}: O rel err {err.max():.3e}"
    assert err.mean() <= 2e-3, f"scale {scale}: O mean err {err.mean():.3e}"
    lerr = np.abs(H.to_f64(lse) - l_ref) / np.maximum(1.0, np.abs(l_ref))
    assert lerr.max() <= 1e-3, f"scale {scale}: LSE rel err {lerr.max():.3e}"
    dq, dk, dv = run_bwd(fa, gpu, o, lse, causal, None, scale)
    g_ref = oracle_mod.attention_bwd(ref["q"], ref["k"], ref["v"], ref["do"], scale, causal=causal)[:3]
    H.assert_grads_close([H.to_f64(x) for x in (dq, dk, dv)], g_ref, f"scale {scale}")


def test_bench_workload_backward_full_size(fa, oracle_mod):
    # The bench's default workload (B=4, H=16, N=4096, d=128) in one launch: one sampled head
    # against the oracle in full, and on every head two identities that hold at any size:
    # sum_j dK_j = 0 (rows of dS sum to zero) and sum_j dV_j = sum_i dO_i (rows of P sum to one).
    B, Hh, N, d = 4, 16, 4096, 128
    check_heads(fa, oracle_mod, B, Hh, N, d, False, None, nheads=1, seed=synth.BASE_SEED + 3)
    gpu, _ = H.make_case(B, Hh, N, d, seed=synth.BASE_SEED + 3)
    scale = 1.0 / np.sqrt(d)
    o, lse = run_fwd(fa, gpu, False, None, scale)
    dq, dk, dv = run_bwd(fa, gpu, o, lse, False, None, scale)
    dk_sum = dk.float().sum(dim=2)
    dv_sum = dv.float().sum(dim=2)
    do_sum = gpu["do"].float().sum(dim=2)
    # bf16 rounding of each dK row (~2^-9 relative) bounds the column sums against the rows' size
    assert (dk_sum.norm(dim=-1) / dk.float().norm(dim=(2, 3))).max().item() < 2e-2
    assert ((dv_sum - do_sum).norm(dim=-1) / do_sum.norm(dim=-1)).max().item() < 2e-2


@pytest.mark.parametrize("B", [65535, 70001])
def test_largest_head_count(fa, oracle_mod, B):
    # B*H = 65535 (one grid dimension's limit) and 70001 (heads spread over two grid
    # dimensions, the last row of CTAs partly past the last head), one 128-row tile per head,
    # forward and backward. Heads are independent: the bulk is seeded device-side random data,
    # and five heads across the range carry synth's draws, which the oracle gets bit for bit.
    N, d, scale = 128, 64, 0.125
    g = torch.Generator(device="cuda").manual_seed(synth.BASE_SEED)
    gpu = {k: torch.randn(B, 1, N, d, device="cuda", dtype=torch.bfloat16, generator=g) for k in ("q", "k", "v", "do")}
    sample = (0, 1, 32767, 65534, B - 1) if B > 65535 else (0, 1, 32767, 65533, 65534)
    small, ref = H.make_case(len(sample), 1, N, d, seed=synth.BASE_SEED + 9)
    for x, b in enumerate(sample):
        for k in gpu:
            gpu[k][b] = small[k][x]
    o, lse = run_fwd(fa, gpu, False, None, scale)
    dq, dk, dv = run_bwd(fa, gpu, o, lse, False, None, scale)
    for x, b in enumerate(sample):
        args = [ref[k][x:x + 1] for k in ("q", "k", "v")]
        o_ref, l_ref = oracle_mod.attention_fwd(*args, scale)
        H.assert_fwd_close(H.to_f64(o[b:b + 1]), H.to_f64(lse[b:b + 1]), o_ref, l_ref, f"head {b}")
        g_ref = oracle_mod.attention_bwd(*args, ref["do"][x:x + 1], scale)[:3]
        H.assert_grads_close([H.to_f64(t[b:b + 1]) for t in (dq, dk, dv)], g_ref, f"head {b}")


def test_fma_pipe_exp2_accuracy(fa):
    # The own cubic exp2 (a compile-time option of the softmax kernels) against exact 2^x and
    # against the special-function unit, over the range softmax exponents take.
    g = torch.Generator().manual_seed(5)
    x = torch.cat([torch.linspace(-120.0, 8.0, 200001, dtype=torch.float64),
                   torch.rand(100000, generator=g, dtype=torch.float64) * 16 - 12]).float()
    poly, sfu = fa.selftest_ex2(x.cuda())
    torch.cuda.synchronize()
    exact = torch.exp2(x.double())
    rel_poly = ((poly.double().cpu() - exact).abs() / exact).max().item()
    rel_sfu = ((sfu.double().cpu() - exact).abs() / exact).max().item()
    assert rel_poly < 1e-4, rel_poly   # fitted bound: 7.5e-5 in fp32 Horner form
    assert rel_sfu < 1e-5, rel_sfu
