"""The FMA-pipe exp2 of the attention kernel: the fitted polynomial and its error bound.

The kernel's ex2_fma_pipe splits x = n + f (n = round(x)) and evaluates a
degree-4 polynomial for 2^f. Here the same steps run in fp32 numpy against
numpy's exp2, and the coefficients written in attn.cu must be the fit's.
"""
import os
import re

import numpy as np

from tile_sparse_video_pack_b200.csrc.fit_exp2_poly import fit, horner_f32

ATTN = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "tile_sparse_video_pack_b200", "csrc", "attn.cu")


def kernel_coefficients():
    src = open(ATTN).read()
    start = src.index("void ex2_fma_pipe")
    body = src[start:src.index("\n}\n", start)]
    vals = [float(v) for v in re.findall(r"f2pack\(([0-9.e-]+)f, \1f\)", body)]
    return np.array(vals[::-1], dtype=np.float32)   # written highest degree first


def emulate(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """The kernel's steps in fp32: clamp, round by 1.5*2^23, polynomial, exponent add."""
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    k = np.float32(12582912.0)
    t = (x + k).astype(np.float32)
    n = (t - k).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = horner_f32(c, f)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_fit_error_bound():
    c, err = fit()
    assert err < 3e-6
    assert np.allclose(c, kernel_coefficients(), rtol=0, atol=0)


def test_emulated_kernel_steps_match_exp2():
    c = kernel_coefficients()
    x = np.concatenate([np.linspace(-124.0, 8.0, 2_000_001), [-0.5, 0.5, 0.0, 7.999]]).astype(np.float32)
    y = emulate(x, c).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 4e-6
    # below the clamp the result is 2^-125, negligible next to the row's largest term (>= 2^-8)
    assert emulate(np.array([-np.inf, -300.0], np.float32), c).max() <= 2.0 ** -124
