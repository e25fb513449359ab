"""Pins for the fp64 oracle: each check is fixed by the mathematics, a library routine or a
hand-derived case, never by the oracle's own formulas retyped.

Mistakes these are meant to catch: a dropped scale, a softmax over the wrong axis, a
missing max-subtraction term, a wrong sign or index in the backward, a transposed operand,
a mask applied to the wrong block or side of the diagonal.
"""
import json
import math
from pathlib import Path

import numpy as np
import pytest
import scipy.special
import torch

import synth

GOLDEN = Path(__file__).parent / "golden"


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def dense_mask(N, causal, mask, bs):
    """Boolean allowed(i, j) matrix built directly from the mask definition."""
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    a = np.ones((N, N), dtype=bool)
    if causal:
        a &= j <= i
    if mask is not None:
        a &= mask[i // bs, j // bs].astype(bool)
    return a


def scipy_attention(q, k, v, scale, allowed):
    """Library-routine reference: scipy.special.softmax / logsumexp per row."""
    B, H, N, d = q.shape
    o = np.zeros_like(q)
    lse = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            s = scale * q[b, h] @ k[b, h].T
            s = np.where(allowed, s, -np.inf)
            p = scipy.special.softmax(s, axis=1)
            o[b, h] = p @ v[b, h]
            lse[b, h] = scipy.special.logsumexp(s, axis=1)
    return o, lse


# ---------------------------------------------------------------------------------------
# Forward pins
# ---------------------------------------------------------------------------------------

def test_golden_two_key_rescale(oracle_mod):
    g = json.loads((GOLDEN / "two_key_rescale.json").read_text())
    q = np.array(g["q"])[None, None]
    k = np.array(g["k"])[None, None]
    v = np.array(g["v"])[None, None]
    o, lse = oracle_mod.attention_fwd(q, k, v, g["scale"])
    np.testing.assert_allclose(o[0, 0], g["expected_o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], g["expected_lse"], rtol=0, atol=1e-14)
    for deferred in (False, True):
        o2, lse2 = oracle_mod.attention_online_fwd(q, k, v, g["scale"], block=1, deferred=deferred)
        np.testing.assert_allclose(o2[0, 0], g["expected_o"], rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse2[0, 0], g["expected_lse"], rtol=0, atol=1e-14)


def test_rows_of_p_sum_to_one_identity_values(oracle_mod):
    # With V = I (N = d) the output rows ARE the probability rows.
    N = 24
    q, k = rnd((1, 1, N, N), 1), rnd((1, 1, N, N), 2)
    v = np.eye(N)[None, None]
    for causal in (False, True):
        o, _ = oracle_mod.attention_fwd(q, k, v, 0.3, causal=causal)
        p = o[0, 0]
        assert np.all(p >= 0)
        np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-14)
        if causal:
            assert np.all(p[np.triu_indices(N, 1)] == 0.0)
        s = 0.3 * q[0, 0] @ k[0, 0].T
        if causal:
            s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
        np.testing.assert_allclose(p, scipy.special.softmax(s, axis=1), rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("use_mask", [False, True])
def test_forward_matches_scipy(oracle_mod, causal, use_mask):
    B, H, N, d, bs = 2, 3, 70, 8, 16
    q, k, v = rnd((B, H, N, d), 3), rnd((B, H, N, d), 4), rnd((B, H, N, d), 5)
    nb = (N + bs - 1) // bs
    mask = synth.bernoulli_block_mask(99, nb, 0.4) if use_mask else None
    o, lse = oracle_mod.attention_fwd(q, k, v, 0.37, causal=causal, mask=mask, mask_bs=bs)
    ro, rl = scipy_attention(q, k, v, 0.37, dense_mask(N, causal, mask, bs))
    np.testing.assert_allclose(o, ro, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, rl, rtol=1e-13, atol=1e-13)


def test_identical_keys_give_mean_of_values(oracle_mod):
    N, d = 40, 6
    q = rnd((1, 1, N, d), 6)
    k = np.tile(rnd((1, d), 7), (N, 1))[None, None]
    v = rnd((1, 1, N, d), 8)
    o, _ = oracle_mod.attention_fwd(q, k, v, 0.5)
    np.testing.assert_allclose(o[0, 0], np.tile(v[0, 0].mean(axis=0), (N, 1)), atol=1e-13)
    oc, _ = oracle_mod.attention_fwd(q, k, v, 0.5, causal=True)
    cummean = np.cumsum(v[0, 0], axis=0) / np.arange(1, N + 1)[:, None]
    np.testing.assert_allclose(oc[0, 0], cummean, atol=1e-13)


def test_dominant_score_selects_its_value_row(oracle_mod):
    # Keys are +-e_t basis directions; one key per row has a score gap of >= 60.
    N, d = 16, 16
    rng = np.random.default_rng(9)
    k = np.eye(d)[None, None] * 1.0
    target = rng.permutation(N)
    q = np.zeros((1, 1, N, d))
    q[0, 0, np.arange(N), target] = 60.0
    v = rnd((1, 1, N, d), 10)
    o, lse = oracle_mod.attention_fwd(q, k, v, 1.0)
    np.testing.assert_allclose(o[0, 0], v[0, 0, target], atol=1e-12)
    # LSE = 60 + ln(1 + (N-1) e^-60)
    np.testing.assert_allclose(lse[0, 0], 60.0 + np.log1p((N - 1) * np.exp(-60.0)), atol=1e-13)


def test_zero_query_lse_counts_allowed_keys(oracle_mod):
    N, d, bs = 96, 4, 16
    q = np.zeros((1, 1, N, d))
    k, v = rnd((1, 1, N, d), 11), rnd((1, 1, N, d), 12)
    o, lse = oracle_mod.attention_fwd(q, k, v, 0.125)
    np.testing.assert_allclose(lse[0, 0], np.log(N), rtol=0, atol=1e-14)
    np.testing.assert_allclose(o[0, 0], np.tile(v[0, 0].mean(0), (N, 1)), atol=1e-13)
    _, lse_c = oracle_mod.attention_fwd(q, k, v, 0.125, causal=True)
    np.testing.assert_allclose(lse_c[0, 0], np.log(np.arange(1, N + 1)), rtol=0, atol=1e-14)
    mask = synth.bernoulli_block_mask(5, N // bs, 0.3)
    _, lse_m = oracle_mod.attention_fwd(q, k, v, 0.125, mask=mask, mask_bs=bs)
    on_per_row = mask.sum(axis=1).repeat(bs)
    np.testing.assert_allclose(lse_m[0, 0], np.log(bs * on_per_row), rtol=0, atol=1e-14)


def test_key_shift_invariance(oracle_mod):
    # Adding c to every key adds scale*q_i.c to row i's scores: O unchanged, LSE shifted.
    N, d, scale = 50, 8, 0.3
    q, k, v = rnd((1, 1, N, d), 13), rnd((1, 1, N, d), 14), rnd((1, 1, N, d), 15)
    c = rnd((d,), 16)
    o1, l1 = oracle_mod.attention_fwd(q, k, v, scale, causal=True)
    o2, l2 = oracle_mod.attention_fwd(q, k + c, v, scale, causal=True)
    np.testing.assert_allclose(o2, o1, atol=1e-12)
    np.testing.assert_allclose(l2, l1 + scale * (q @ c), atol=1e-12)


def test_fully_masked_row_is_zero(oracle_mod):
    N, d, bs = 8, 4, 4
    mask = np.array([[0, 0], [1, 1]], dtype=np.uint8)  # rows 0..3 see nothing
    q, k, v = rnd((1, 1, N, d), 17), rnd((1, 1, N, d), 18), rnd((1, 1, N, d), 19)
    o, lse = oracle_mod.attention_fwd(q, k, v, 0.5, mask=mask, mask_bs=bs)
    assert np.all(o[0, 0, :4] == 0.0) and np.all(np.isneginf(lse[0, 0, :4]))
    dq, dk, dv, _ = oracle_mod.attention_bwd(q, k, v, rnd((1, 1, N, d), 20), 0.5, mask=mask, mask_bs=bs)
    assert np.all(np.isfinite(dq)) and np.all(dq[0, 0, :4] == 0.0)


@pytest.mark.parametrize("block", [1, 3, 16, 128])
@pytest.mark.parametrize("deferred", [False, True])
def test_online_equals_three_pass(oracle_mod, block, deferred):
    B, H, N, d, bs = 1, 2, 300, 16, 32
    q, k, v = rnd((B, H, N, d), 21, 2.0), rnd((B, H, N, d), 22, 2.0), rnd((B, H, N, d), 23)
    mask = synth.bernoulli_block_mask(7, (N + bs - 1) // bs, 0.5)
    for causal, m in ((False, None), (True, None), (True, mask)):
        o3, l3 = oracle_mod.attention_fwd(q, k, v, 0.25, causal=causal, mask=m, mask_bs=bs)
        oo, lo = oracle_mod.attention_online_fwd(q, k, v, 0.25, block=block, deferred=deferred,
                                                 causal=causal, mask=m, mask_bs=bs)
        np.testing.assert_allclose(oo, o3, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lo, l3, rtol=0, atol=1e-13)


def test_masks_reduce_to_dense(oracle_mod):
    N, d, bs = 64, 8, 16
    nb = N // bs
    q, k, v = rnd((1, 1, N, d), 24), rnd((1, 1, N, d), 25), rnd((1, 1, N, d), 26)
    dense = oracle_mod.attention_fwd(q, k, v, 0.3)
    ones = oracle_mod.attention_fwd(q, k, v, 0.3, mask=np.ones((nb, nb), np.uint8), mask_bs=bs)
    assert np.array_equal(dense[0], ones[0]) and np.array_equal(dense[1], ones[1])
    # Diagonal-only mask == independent dense attention inside each chunk.
    o_diag, l_diag = oracle_mod.attention_fwd(q, k, v, 0.3, mask=np.eye(nb, dtype=np.uint8), mask_bs=bs)
    for c in range(nb):
        sl = slice(c * bs, (c + 1) * bs)
        oc, lc = oracle_mod.attention_fwd(q[:, :, sl], k[:, :, sl], v[:, :, sl], 0.3)
        np.testing.assert_allclose(o_diag[:, :, sl], oc, atol=1e-14)
        np.testing.assert_allclose(l_diag[:, :, sl], lc, atol=1e-14)
    # Causal row i == dense attention of query i over keys 0..i.
    o_c, l_c = oracle_mod.attention_fwd(q, k, v, 0.3, causal=True)
    for i in (0, 1, 17, 63):
        oi, li = oracle_mod.attention_fwd_rows(q[0, 0, :i + 1], k[0, 0, :i + 1], v[0, 0, :i + 1], [i], 0.3)
        np.testing.assert_allclose(o_c[0, 0, i], oi[0], atol=1e-14)
        np.testing.assert_allclose(l_c[0, 0, i], li[0], atol=1e-14)


def test_rows_variant_matches_full(oracle_mod):
    N, d = 200, 16
    q, k, v = rnd((1, 1, N, d), 27), rnd((1, 1, N, d), 28), rnd((1, 1, N, d), 29)
    mask = synth.bernoulli_block_mask(3, 4, 0.5)
    o, l = oracle_mod.attention_fwd(q, k, v, 0.2, causal=True, mask=mask, mask_bs=64)
    rows = [0, 5, 63, 64, 130, 199]
    orow, lrow = oracle_mod.attention_fwd_rows(q[0, 0], k[0, 0], v[0, 0], rows, 0.2, causal=True,
                                               mask=mask, mask_bs=64)
    np.testing.assert_array_equal(orow, o[0, 0, rows])
    np.testing.assert_array_equal(lrow, l[0, 0, rows])


# ---------------------------------------------------------------------------------------
# Backward pins
# ---------------------------------------------------------------------------------------

def torch_reference_grads(q, k, v, do, scale, allowed):
    """torch.autograd in fp64 on the plain dense formula (a library routine, not the oracle)."""
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    s = scale * tq @ tk.transpose(-1, -2)
    s = s.masked_fill(~torch.tensor(allowed), float("-inf"))
    o = torch.softmax(s, dim=-1) @ tv
    o.backward(torch.tensor(do, dtype=torch.float64))
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy(), o.detach().numpy()


@pytest.mark.parametrize("causal,use_mask", [(False, False), (True, False), (False, True), (True, True)])
def test_backward_matches_torch_autograd(oracle_mod, causal, use_mask):
    B, H, N, d, bs = 2, 2, 48, 8, 16
    q, k, v, do = (rnd((B, H, N, d), s) for s in (30, 31, 32, 33))
    mask = synth.bernoulli_block_mask(11, N // bs, 0.5) if use_mask else None
    allowed = dense_mask(N, causal, mask, bs)
    dq, dk, dv, D = oracle_mod.attention_bwd(q, k, v, do, 0.35, causal=causal, mask=mask, mask_bs=bs)
    tq, tk, tv, to = torch_reference_grads(q, k, v, do, 0.35, allowed)
    np.testing.assert_allclose(dq, tq, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dk, tk, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dv, tv, rtol=1e-11, atol=1e-12)
    # D_i = sum_j P_ij dP_ij must equal dO_i . O_i
    np.testing.assert_allclose(D, (do * to).sum(-1), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("N,d", [(5, 3), (8, 4), (16, 8)])
@pytest.mark.parametrize("causal,use_mask", [(False, False), (True, False), (True, True)])
def test_backward_matches_finite_differences(oracle_mod, N, d, causal, use_mask):
    scale, h, bs = 0.6, 1e-6, 4
    q, k, v, do = (rnd((1, 1, N, d), s) for s in (40, 41, 42, 43))
    nb = (N + bs - 1) // bs
    mask = synth.bernoulli_block_mask(12, nb, 0.5) if use_mask else None

    def loss(q_, k_, v_):
        o, _ = oracle_mod.attention_fwd(q_, k_, v_, scale, causal=causal, mask=mask, mask_bs=bs)
        return float((o * do).sum())

    dq, dk, dv, _ = oracle_mod.attention_bwd(q, k, v, do, scale, causal=causal, mask=mask, mask_bs=bs)
    for idx, (x, g) in enumerate(((q, dq), (k, dk), (v, dv))):
        num = np.zeros_like(x)
        for pos in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[pos] += h
            xm[pos] -= h
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[idx], args_m[idx] = xp, xm
            num[pos] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.linalg.norm(num - g) / max(np.linalg.norm(g), 1e-30)
        assert err < 1e-7, (idx, err)


def test_backward_sum_identities(oracle_mod):
    B, H, N, d = 1, 3, 100, 16
    q, k, v, do = (rnd((B, H, N, d), s) for s in (50, 51, 52, 53))
    for causal in (False, True):
        dq, dk, dv, D = oracle_mod.attention_bwd(q, k, v, do, 0.25, causal=causal)
        o, _ = oracle_mod.attention_fwd(q, k, v, 0.25, causal=causal)
        # softmax is shift-invariant per row -> sum over keys of dK vanishes
        np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-11)
        # rows of P sum to one -> sum over keys of dV equals the sum over queries of dO
        np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), atol=1e-11)
        np.testing.assert_allclose(D, (do * o).sum(-1), atol=1e-12)


def test_bf16_inputs_are_exact_in_fp64():
    bits = synth.normal_bf16(123, 1000)
    f = synth.bf16_bits_to_f32(bits).astype(np.float64)
    assert np.array_equal(synth.f32_to_bf16_bits(f.astype(np.float32)), bits)
    assert abs(f.mean()) < 0.15 and abs(f.std() - 1.0) < 0.1


# ---------------------------------------------------------------------------------------
# General shapes (N_q queries against N_k keys) and the split-KV combine
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_general_shapes_reduce_to_square(oracle_mod, causal):
    # N_q = N_k: the offset is zero and the result is the square oracle's
    q, k, v = rnd((1, 2, 45, 8), 60), rnd((1, 2, 45, 8), 61), rnd((1, 2, 45, 8), 62)
    o1, l1 = oracle_mod.attention_fwd_qk(q, k, v, 0.4, causal=causal)
    o2, l2 = oracle_mod.attention_fwd(q, k, v, 0.4, causal=causal)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_bottom_right_causal_is_the_suffix_of_the_square_problem(oracle_mod):
    # The last N_q rows of a square causal problem see exactly the keys the bottom-right
    # alignment gives N_q queries against the same N_k keys.
    N, nq = 53, 7
    q, k, v = rnd((2, 1, N, 8), 63), rnd((2, 1, N, 8), 64), rnd((2, 1, N, 8), 65)
    o_sq, l_sq = oracle_mod.attention_fwd(q, k, v, 0.3, causal=True)
    o, l = oracle_mod.attention_fwd_qk(q[:, :, N - nq:], k, v, 0.3, causal=True)
    np.testing.assert_allclose(o, o_sq[:, :, N - nq:], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(l, l_sq[:, :, N - nq:], rtol=1e-13, atol=1e-14)


def test_general_shapes_match_scipy(oracle_mod):
    # N_q != N_k against a library softmax over the explicitly built allowed matrix
    nq, nk, d = 9, 40, 6
    q, k, v = rnd((1, 2, nq, d), 66), rnd((1, 2, nk, d), 67), rnd((1, 2, nk, d), 68)
    for causal in (False, True):
        o, l = oracle_mod.attention_fwd_qk(q, k, v, 0.5, causal=causal)
        i = np.arange(nq)[:, None]
        j = np.arange(nk)[None, :]
        allowed = (j <= i + (nk - nq)) if causal else np.ones((nq, nk), dtype=bool)
        for h in range(2):
            s = np.where(allowed, 0.5 * q[0, h] @ k[0, h].T, -np.inf)
            np.testing.assert_allclose(o[0, h], scipy.special.softmax(s, axis=1) @ v[0, h], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(l[0, h], scipy.special.logsumexp(s, axis=1), rtol=1e-13, atol=1e-13)


def test_more_queries_than_keys_causal_rows_see_nothing(oracle_mod):
    # bottom-right alignment with N_q > N_k: the first N_q - N_k rows have no visible key
    q, k, v = rnd((1, 1, 10, 4), 69), rnd((1, 1, 6, 4), 70), rnd((1, 1, 6, 4), 71)
    o, l = oracle_mod.attention_fwd_qk(q, k, v, 0.5, causal=True)
    assert np.all(o[0, 0, :4] == 0) and np.all(np.isneginf(l[0, 0, :4]))
    assert np.all(np.isfinite(l[0, 0, 4:]))


def test_split_keys_and_merge_by_lse_equals_full(oracle_mod):
    # The split-KV forward computes (O_s, LSE_s) on key chunks and combines them with
    # LSE = log sum_s exp(LSE_s), O = sum_s exp(LSE_s - LSE) O_s: the online normaliser's
    # combine step, here checked against the unsplit result in fp64.
    nq, nk, d = 5, 300, 8
    q, k, v = rnd((1, 2, nq, d), 72), rnd((1, 2, nk, d), 73), rnd((1, 2, nk, d), 74)
    o_full, l_full = oracle_mod.attention_fwd_qk(q, k, v, 0.35)
    cuts = [0, 64, 65, 190, 300]  # uneven chunks, one of a single key
    parts = [oracle_mod.attention_fwd_qk(q, k[:, :, a:b], v[:, :, a:b], 0.35) for a, b in zip(cuts, cuts[1:])]
    ls = np.stack([p[1] for p in parts])
    lse = scipy.special.logsumexp(ls, axis=0)
    o = sum(np.exp(p[1] - lse)[..., None] * p[0] for p in parts)
    np.testing.assert_allclose(o, o_full, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, l_full, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------------------------------
# General-shape backward (the gradient of attention_fwd_qk)
# ---------------------------------------------------------------------------------------

def allowed_qk(nq, nk, causal):
    """Bottom-right alignment built directly from its definition: j <= i + (N_k - N_q)."""
    i = np.arange(nq)[:, None]
    j = np.arange(nk)[None, :]
    return (j <= i + (nk - nq)) if causal else np.ones((nq, nk), dtype=bool)


@pytest.mark.parametrize("nq,nk,causal", [(9, 40, False), (9, 40, True), (33, 20, False), (20, 20, True)])
def test_general_backward_matches_torch_autograd(oracle_mod, nq, nk, causal):
    d = 6
    q, do = rnd((2, 2, nq, d), 80), rnd((2, 2, nq, d), 81)
    k, v = rnd((2, 2, nk, d), 82), rnd((2, 2, nk, d), 83)
    dq, dk, dv, D = oracle_mod.attention_bwd_qk(q, k, v, do, 0.45, causal=causal)
    tq, tk, tv, to = torch_reference_grads(q, k, v, do, 0.45, allowed_qk(nq, nk, causal))
    np.testing.assert_allclose(dq, tq, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dk, tk, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dv, tv, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(D, (do * to).sum(-1), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("nq,nk,causal", [(3, 7, True), (7, 5, True), (4, 9, False)])
def test_general_backward_matches_finite_differences(oracle_mod, nq, nk, causal):
    # (7, 5, causal): rows 0 and 1 see no key; their output is the constant 0.
    d, scale, h = 3, 0.7, 1e-6
    q, do = rnd((1, 1, nq, d), 84), rnd((1, 1, nq, d), 85)
    k, v = rnd((1, 1, nk, d), 86), rnd((1, 1, nk, d), 87)

    def loss(q_, k_, v_):
        o, _ = oracle_mod.attention_fwd_qk(q_, k_, v_, scale, causal=causal)
        return float((o * do).sum())

    grads = oracle_mod.attention_bwd_qk(q, k, v, do, scale, causal=causal)[:3]
    for idx, (x, g) in enumerate(zip((q, k, v), grads)):
        num = np.zeros_like(x)
        for pos in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[pos] += h
            xm[pos] -= h
            args_p, args_m = [q, k, v], [q, k, v]
            args_p[idx], args_m[idx] = xp, xm
            num[pos] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.linalg.norm(num - g) / max(np.linalg.norm(g), 1e-30)
        assert err < 1e-7, (idx, err)


@pytest.mark.parametrize("causal", [False, True])
def test_general_backward_reduces_to_square(oracle_mod, causal):
    q, k, v, do = (rnd((1, 2, 45, 8), s) for s in (88, 89, 90, 91))
    a = oracle_mod.attention_bwd_qk(q, k, v, do, 0.4, causal=causal)
    b = oracle_mod.attention_bwd(q, k, v, do, 0.4, causal=causal)
    for x, y in zip(a, b):  # dK, dV: per-thread partial sums, added in a schedule-dependent order
        np.testing.assert_allclose(x, y, rtol=1e-12, atol=1e-14)


def test_general_backward_is_the_suffix_of_the_square_problem(oracle_mod):
    # A square causal problem whose upstream gradient is zero on all but the last nq rows
    # has the same dK and dV, and the same dQ on those rows, as nq bottom-right-aligned queries
    # against all N keys (and dQ = 0 on the other rows).
    N, nq, d = 50, 11, 5
    q, k, v = rnd((1, 2, N, d), 92), rnd((1, 2, N, d), 93), rnd((1, 2, N, d), 94)
    do = rnd((1, 2, N, d), 95)
    do[:, :, :N - nq] = 0.0
    dq_sq, dk_sq, dv_sq, _ = oracle_mod.attention_bwd(q, k, v, do, 0.3, causal=True)
    dq, dk, dv, _ = oracle_mod.attention_bwd_qk(q[:, :, N - nq:], k, v, do[:, :, N - nq:], 0.3, causal=True)
    np.testing.assert_allclose(dq, dq_sq[:, :, N - nq:], rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(dq_sq[:, :, :N - nq], 0.0)
    np.testing.assert_allclose(dk, dk_sq, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dv, dv_sq, rtol=1e-12, atol=1e-13)


def test_general_backward_rows_that_see_nothing(oracle_mod):
    # N_q > N_k, causal: the first N_q - N_k rows see no key. Their dQ is exactly zero and
    # their upstream gradient reaches neither dK nor dV.
    nq, nk, d = 12, 5, 4
    q, k, v, do = rnd((1, 1, nq, d), 96), rnd((1, 1, nk, d), 97), rnd((1, 1, nk, d), 98), rnd((1, 1, nq, d), 99)
    dq, dk, dv, D = oracle_mod.attention_bwd_qk(q, k, v, do, 0.5, causal=True)
    assert np.all(dq[0, 0, :nq - nk] == 0) and np.all(D[0, 0, :nq - nk] == 0)
    do2 = do.copy()
    do2[:, :, :nq - nk] = rnd((1, 1, nq - nk, d), 100) * 7.0
    _, dk2, dv2, _ = oracle_mod.attention_bwd_qk(q, k, v, do2, 0.5, causal=True)
    np.testing.assert_allclose(dk, dk2, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(dv, dv2, rtol=1e-13, atol=1e-15)
