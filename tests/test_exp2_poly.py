"""The FMA-pipe exp2 used by the attention softmax: its cubic stays within its
stated relative-error bound (checked in fp32 arithmetic, like the kernel), and
the coefficients compiled into the kernel are the ones the fitting script gives."""
import os
import re
import runpy

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "block_sparse_attention_sdl_b200", "csrc")


def test_cubic_error_bound_and_kernel_constants():
    mod = runpy.run_path(os.path.join(CSRC, "exp2_poly.py"))
    c = [np.float32(x) for x in mod["fit"]()]
    err = mod["max_rel_error"](c)
    assert err < 1e-4  # far below bf16's 2^-9 rounding of the weights
    src = open(os.path.join(CSRC, "ptx.cuh")).read()
    consts = [float.fromhex(h) for h in re.findall(r"(0x1\.[0-9a-f]+p-?\d+)f", src)]
    for ci in c:
        assert any(abs(float(ci) - k) <= abs(float(ci)) * 2 ** -23 for k in consts), float(ci)


def test_range_reduction_matches_exp2():
    # emulate exp2_poly in float32: x = n + f with n from the 1.5*2^23 rounding trick
    mod = runpy.run_path(os.path.join(CSRC, "exp2_poly.py"))
    c = [np.float32(x) for x in mod["fit"]()]
    x = np.concatenate([np.linspace(-125, 8, 200001), [-0.5, 0.5, 0.0, -1.0, 7.999]]).astype(np.float32)
    C = np.float32(12582912.0)
    t = (x + C).astype(np.float32)
    n = (t - C).astype(np.float32)
    f = (x - n).astype(np.float32)
    assert np.all(np.abs(f) <= 0.5)
    p = np.float32(c[3])
    for ci in (c[2], c[1], c[0]):
        p = (p * f + ci).astype(np.float32)
    j = t.view(np.int32) - np.int32(0x4B400000)
    y = (p.view(np.int32) + (j << 23)).view(np.float32).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 1e-4
