"""The allocation-free selection entry point, called through the C ABI.

sdl_select_mask_noalloc serves callers that cannot allocate device memory (a
device-memory pool's own callbacks, or a process that reserves its memory up
front and forbids cudaMalloc later): its scratch is a fixed array inside the
library.  It must give exactly the mask of sdl_select_mask, also on a second
call that finds the array holding the first call's leftovers.  This file is
collected last so that a run stopping at the first failure has run every other
test first.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

sdl = pytest.importorskip("block_sparse_attention_sdl_b200")


def _noalloc():
    f = sdl.lib().sdl_select_mask_noalloc
    f.argtypes = [ctypes.c_void_p, ctypes.POINTER(sdl.Shape), ctypes.c_double, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def _shape(B, H, L, block):
    s = sdl.Shape()
    s.B, s.H, s.H_kv, s.L, s.d, s.block, s.dtype = B, H, H, L, 64, block, sdl.SDL_FP32
    return s


@pytest.mark.parametrize("B,H,nb,block,sparsity", [(1, 32, 128, 64, 0.9), (2, 4, 32, 64, 0.8),
                                                   (1, 32, 512, 128, 0.95)])
def test_noalloc_matches_workspace_entry_point_twice(B, H, nb, block, sparsity):
    torch.manual_seed(nb + H)
    f = _noalloc()
    stream = torch.cuda.current_stream().cuda_stream
    shape = _shape(B, H, nb * block, block)
    for call in range(2):
        logits = torch.randn(B, H, nb, nb, device="cuda") * (1.0 + call)
        scores = torch.softmax(logits, dim=-1).contiguous()
        rp_ref, ci_ref, m_ref = sdl.select_mask(scores, sparsity, block, nb * block,
                                                want_mask=True)
        total = ci_ref.numel()
        rp = torch.full_like(rp_ref, -1)
        ci = torch.full_like(ci_ref, -1)
        m = torch.full_like(m_ref, 7)
        rc = f(scores.data_ptr(), ctypes.byref(shape), sparsity, rp.data_ptr(), ci.data_ptr(),
               total, m.data_ptr(), stream)
        assert rc == sdl.SDL_OK
        torch.cuda.synchronize()
        assert torch.equal(rp, rp_ref), call
        assert torch.equal(ci, ci_ref), call
        assert torch.equal(m, m_ref), call


def test_noalloc_rejects_problems_beyond_its_scratch():
    f = _noalloc()
    big = _shape(16, 64, 65536, 64)  # 1M query-block rows: far more than 2 MiB of scratch
    assert sdl.select_workspace_bytes(big) > (2 << 20)
    P = ctypes.c_void_p
    rc = f(P(256), ctypes.byref(big), 0.99, P(256), P(256), 1 << 40, None, None)
    assert rc == sdl.SDL_ERR_WORKSPACE
    small = _shape(1, 2, 512, 64)
    rc = f(P(256), ctypes.byref(small), 0.5, P(256), P(256), 3, None, None)
    assert rc == sdl.SDL_ERR_CAPACITY
