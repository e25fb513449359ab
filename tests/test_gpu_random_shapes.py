"""Randomised parity: seeded random problem shapes (sequence lengths with ragged tails, N_q
against N_k, every head dimension, causal or block-sparse masks, bf16 and fp16), each run through
the C ABI and compared with the fp64 oracle in full at the parity bars. The shapes are drawn
from a fixed seed, so every run checks the same cases."""
import numpy as np
import pytest
import torch

import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu


def draw_cases(n=24, seed=20261203):
    rng = np.random.default_rng(seed)
    cases = []
    for x in range(n):
        d = int(rng.choice([64, 128, 256]))
        square = x % 3 != 2
        nq = int(rng.integers(1, 700))
        nk = nq if square else int(rng.integers(1, 900))
        causal = bool(rng.integers(0, 2))
        mask = square and not causal and bool(rng.integers(0, 3) == 0)
        dtype = "f16" if rng.integers(0, 4) == 0 else "bf16"
        B, Hh = int(rng.integers(1, 3)), int(rng.integers(1, 3))
        cases.append((x, B, Hh, nq, nk, d, causal, mask, dtype))
    return cases


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import exact_attention_110_b200 as fa
    fa.library()
    return fa


@pytest.mark.parametrize("x,B,Hh,nq,nk,d,causal,mask,dtype", draw_cases())
def test_random_shape(fa, oracle_mod, x, B, Hh, nq, nk, d, causal, mask, dtype):
    seed = synth.BASE_SEED + 1000 + 17 * x
    scale = 1.0 / np.sqrt(d)
    what = f"case {x}: B={B} H={Hh} Nq={nq} Nk={nk} d={d} causal={causal} mask={mask} {dtype}"
    if nq == nk:
        gpu, ref = H.make_case(B, Hh, nq, d, seed=seed, dtype=dtype)
        m = synth.bernoulli_block_mask(seed, (nq + 127) // 128, p=0.4) if mask else None
        mt = None if m is None else torch.from_numpy(m).cuda()
        o, lse = fa.forward(gpu["q"], gpu["k"], gpu["v"], causal=causal, block_mask=mt, scale=scale)
        dq, dk, dv = fa.backward(gpu["q"], gpu["k"], gpu["v"], o, gpu["do"], lse, causal=causal, block_mask=mt,
                                 scale=scale)
        torch.cuda.synchronize()
        assert fa.last_device_status() == 0
        o_ref, l_ref = oracle_mod.attention_fwd(ref["q"], ref["k"], ref["v"], scale, causal=causal, mask=m)
        g_ref = oracle_mod.attention_bwd(ref["q"], ref["k"], ref["v"], ref["do"], scale, causal=causal, mask=m)[:3]
    else:
        gq, rq = H.make_case(B, Hh, nq, d, seed=seed, dtype=dtype)
        gk, rk = H.make_case(B, Hh, nk, d, seed=seed + 500, with_do=False, dtype=dtype)
        o, lse = fa.forward_decode(gq["q"], gk["k"], gk["v"], causal=causal, scale=scale)
        dq, dk, dv = fa.backward_qk(gq["q"], gk["k"], gk["v"], o, gq["do"], lse, causal=causal, scale=scale)
        torch.cuda.synchronize()
        assert fa.last_device_status() == 0
        o_ref, l_ref = oracle_mod.attention_fwd_qk(rq["q"], rk["k"], rk["v"], scale, causal=causal)
        g_ref = oracle_mod.attention_bwd_qk(rq["q"], rk["k"], rk["v"], rq["do"], scale, causal=causal)[:3]
    H.assert_fwd_close(H.to_f64(o), H.to_f64(lse), o_ref, l_ref, what)
    H.assert_grads_close([H.to_f64(t) for t in (dq, dk, dv)], g_ref, what)
