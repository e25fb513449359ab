"""The FMA-pipe exp2's cubic: its coefficients in csrc/ptx.cuh are exactly what the committed
fitting script (Lawson's iteratively reweighted least squares for the minimax relative error
on [-0.5, 0.5]) prints, and the fp32 Horner evaluation stays within its bound. The GPU side
(test_fma_pipe_exp2_accuracy) checks the kernels' own evaluation against exact 2^x."""
import re
from pathlib import Path

import numpy as np

from exact_attention_110_b200 import fit_ex2_poly

PTX = Path(__file__).resolve().parent.parent / "exact_attention_110_b200" / "csrc" / "ptx.cuh"


def header_coefficients():
    text = PTX.read_text()
    return np.array([float(re.search(rf"kEx2C{k} = ([0-9.eE+-]+)f;", text).group(1)) for k in range(4)],
                    dtype=np.float32)


def test_header_constants_come_from_the_fit():
    np.testing.assert_array_equal(header_coefficients(), fit_ex2_poly.fit())


def test_fit_is_equioscillating_and_within_bound():
    c = fit_ex2_poly.fit()
    assert fit_ex2_poly.max_rel_error_fp32(c) < 8e-5
    # minimax in real arithmetic: the relative error reaches its extreme at five points with
    # alternating signs (degree 3 + 2), both interval ends included
    f = np.linspace(-0.5, 0.5, 20001)
    e = np.polyval(c.astype(np.float64)[::-1], f) / np.exp2(f) - 1.0
    peak = np.abs(e).max()
    assert abs(abs(e[0]) - peak) < 0.02 * peak and abs(abs(e[-1]) - peak) < 0.02 * peak
    big = np.abs(e) > 0.98 * peak
    signs = np.sign(e[big])
    assert np.count_nonzero(np.diff(signs)) >= 4
