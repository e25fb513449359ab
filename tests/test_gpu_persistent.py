"""GPU tests aimed at the persistent backward (problems with at most 8 query tiles, d <= 128):
CTAs that walk several (head, key tile) items taken from a counter in the workspace."""
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


@pytest.mark.parametrize("causal", [False, True])
def test_back_to_back_launches_on_one_workspace(fa, oracle_mod, causal):
    # 8 x 32 heads x 4 key tiles = 1024 items for 148 persistent CTAs. The item counter lives in
    # the workspace: the preprocess zeroes it, and the last CTA of each launch zeroes it again,
    # so a second launch of the main kernel without a new preprocess walks every item again and
    # writes the same dK and dV bit for bit.
    B, Hh, N, d = 8, 32, 512, 64
    gpu, ref = H.make_case(B, Hh, N, d, seed=synth.BASE_SEED + 211)
    scale = 1.0 / np.sqrt(d)
    o, lse = fa.forward(gpu["q"], gpu["k"], gpu["v"], causal=causal, scale=scale)
    ws = fa.bwd_preprocess(o, gpu["do"], lse, scale=scale)
    dk1, dv1 = fa.bwd_main(gpu["q"], gpu["k"], gpu["v"], gpu["do"], ws, causal=causal, scale=scale)
    dk2, dv2 = fa.bwd_main(gpu["q"], gpu["k"], gpu["v"], gpu["do"], ws, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.last_device_status() == 0
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    # and both equal the one-call backward, whose dQ and dK, dV match the oracle on two heads
    dq, dk, dv = fa.backward(gpu["q"], gpu["k"], gpu["v"], o, gpu["do"], lse, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert torch.equal(dk, dk1) and torch.equal(dv, dv1)
    for (b, h) in ((0, 0), (B - 1, Hh - 1)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        args = [ref[x][sl] for x in ("q", "k", "v")]
        g_ref = oracle_mod.attention_bwd(*args, ref["do"][sl], scale, causal=causal)[:3]
        H.assert_grads_close([H.to_f64(x)[sl] for x in (dq, dk, dv)], g_ref, f"head {b},{h}")


@pytest.mark.parametrize("d", [64, 128])
def test_block_mask_that_empties_a_key_tile(fa, oracle_mod, d):
    # Key tile 2 is off for every query tile: its items have no query tile to walk, and their
    # dK and dV must come out as exact zeros while the persistent CTAs carry on to later items
    # (at d = 64 the S^T buffers alternate by active tile, which such items do not advance).
    B, Hh, N = 2, 80, 512
    nb = N // 128
    mask = np.ones((nb, nb), np.uint8)
    mask[:, 2] = 0
    gpu, ref = H.make_case(B, Hh, N, d, seed=synth.BASE_SEED + 223)
    scale = 1.0 / np.sqrt(d)
    mt = torch.from_numpy(mask).cuda()
    o, lse = fa.forward(gpu["q"], gpu["k"], gpu["v"], block_mask=mt, scale=scale)
    dq, dk, dv = fa.backward(gpu["q"], gpu["k"], gpu["v"], o, gpu["do"], lse, block_mask=mt, scale=scale)
    torch.cuda.synchronize()
    assert fa.last_device_status() == 0
    assert not dk[:, :, 256:384].any() and not dv[:, :, 256:384].any()
    for (b, h) in ((0, 3), (1, 77)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        args = [ref[x][sl] for x in ("q", "k", "v")]
        o_ref, lse_ref = oracle_mod.attention_fwd(*args, scale, mask=mask)
        H.assert_fwd_close(H.to_f64(o)[sl], H.to_f64(lse)[sl], o_ref, lse_ref, f"head {b},{h}")
        g_ref = oracle_mod.attention_bwd(*args, ref["do"][sl], scale, mask=mask)[:3]
        H.assert_grads_close([H.to_f64(x)[sl] for x in (dq, dk, dv)], g_ref, f"head {b},{h}")
