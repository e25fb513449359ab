"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device memory.

Some callers of this library cannot call cudaMalloc: hosts that own every device allocation
and forbid allocating inside their execution callbacks, or real-time loops that must not
allocate after start-up. fa_bwd_noalloc serves them by taking its workspace from a fixed
array inside the library. This test calls it through the C ABI and checks that two calls in
a row give the same gradients as fa_bwd with a caller workspace (the second call runs on
whatever the first left in the shared array).

The file name sorts last so that a `-x` run has already run every other test if this fails.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu


def test_noalloc_backward_matches_workspace_backward():
    if not torch.cuda.is_available():
        pytest.fail("GPU test needs a CUDA device")
    import exact_attention_110_b200 as fa

    lib = fa.library()
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.fa_bwd_noalloc.restype = i32
    lib.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, i32, vp, vp]

    for (B, Hh, N, d, causal) in ((2, 4, 512, 64, False), (1, 2, 1024, 128, True)):
        gpu, _ = H.make_case(B, Hh, N, d, seed=synth.BASE_SEED + 5)
        q, k, v, do = gpu["q"], gpu["k"], gpu["v"], gpu["do"]
        scale = 1.0 / np.sqrt(d)
        o, lse = fa.forward(q, k, v, causal=causal, scale=scale)
        ref = fa.backward(q, k, v, o, do, lse, causal=causal, scale=scale)
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        for _ in range(2):
            dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
            st = lib.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                                    lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hh, N, d,
                                    scale, int(causal), None, stream)
            assert st == 0, lib.fa_status_string(st)
            torch.cuda.synchronize()
            assert fa.last_device_status() == 0
            H.assert_grads_close([H.to_f64(x) for x in (dq, dk, dv)], [H.to_f64(x) for x in ref],
                                 f"noalloc vs workspace {B, Hh, N, d, causal}")

    # Sizes beyond the fixed array are refused with FA_ERR_WORKSPACE, before any launch.
    st = lib.fa_bwd_noalloc(16, 16, 16, 16, 16, 16, 16, 16, 16, 64, 16, 4096, 128, 0.1, 0, None, None)
    assert st == 5
