"""The C-ABI library: loads without a GPU, exports every declared symbol, and
validates arguments on the host (no call here reaches the GPU)."""
import ctypes
import os
import re

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sdl.h")

sdl = pytest.importorskip("block_sparse_attention_sdl_b200")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(sdl_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 10
    lib = sdl.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(sdl.EXPORTS)


def _shape(B=1, H=32, Hkv=32, L=8192, d=128, block=64, dtype=0):
    s = sdl.Shape()
    s.B, s.H, s.H_kv, s.L, s.d, s.block, s.dtype = B, H, Hkv, L, d, block, dtype
    for arr in (s.q_strides, s.k_strides, s.v_strides, s.o_strides):
        arr[:] = (L * H * d, H * d, d)
    return s


@pytest.mark.parametrize("H,L,block,s", [(2, 512, 64, 0.5), (32, 2048, 64, 0.8),
                                         (32, 8192, 64, 0.9), (28, 16384, 64, 0.9),
                                         (32, 65536, 128, 0.95), (4, 1024, 128, 0.3)])
def test_budget_matches_oracle(H, L, block, s):
    shp = _shape(H=H, Hkv=H if H != 28 else 4, L=L, block=block)
    nb = L // block
    assert sdl.mask_budget(shp, s) == oracle.budget(H, nb, s)
    shp.B = 3
    assert sdl.mask_budget(shp, s) == 3 * oracle.budget(H, nb, s)


def test_budget_rejects_bad_sparsity():
    shp = _shape(H=2, Hkv=2, L=512)
    for s in (1.0, -0.01, float("nan"), 0.9):  # 0.9 keeps 13 < 16 diagonal blocks
        assert sdl.mask_budget(shp, s) == -1


def test_shape_validation():
    lib = sdl.lib()
    assert sdl.scores_workspace_bytes(_shape()) > 0
    assert sdl.select_workspace_bytes(_shape()) > 0
    for bad in (_shape(block=96), _shape(d=96), _shape(L=8192 + 32), _shape(L=8192 + 64, block=128), _shape(Hkv=5),
                _shape(B=0), _shape(dtype=7), _shape(L=131072)):
        assert sdl.select_workspace_bytes(bad) == 0
        assert sdl.mask_budget(bad, 0.5) == -1
    P = ctypes.c_void_p
    # null pointers and bad shapes are refused before any CUDA call
    rc = lib.sdl_dense_attn(None, None, None, ctypes.byref(_shape()), 0.0, None, None, None)
    assert rc == sdl.SDL_ERR_INVALID_ARG
    rc = lib.sdl_dense_attn(P(16), P(16), P(16), ctypes.byref(_shape(block=96)), 0.0, P(16),
                            None, None)
    assert rc == sdl.SDL_ERR_UNSUPPORTED
    rc = lib.sdl_dense_attn(P(8), P(16), P(16), ctypes.byref(_shape()), 0.0, P(16), None, None)
    assert rc == sdl.SDL_ERR_INVALID_ARG  # misaligned q
    bad_stride = _shape()
    bad_stride.k_strides[1] = 4100
    rc = lib.sdl_dense_attn(P(16), P(16), P(16), ctypes.byref(bad_stride), 0.0, P(16), None, None)
    assert rc == sdl.SDL_ERR_INVALID_ARG
    rc = lib.sdl_sparse_attn(P(16), P(16), P(16), ctypes.byref(_shape()), None, None, 0.0,
                             P(16), None, None)
    assert rc == sdl.SDL_ERR_INVALID_ARG
    rc = lib.sdl_block_scores(P(16), P(16), ctypes.byref(_shape()), 0.0, P(16), None, 0, None)
    assert rc == sdl.SDL_ERR_WORKSPACE
    shp = _shape(H=2, Hkv=2, L=512)
    rc = lib.sdl_select_mask(P(16), ctypes.byref(shp), 0.5, P(16), P(16), 10, None, P(16),
                             1 << 20, None)
    assert rc == sdl.SDL_ERR_CAPACITY
    rc = lib.sdl_select_mask(P(16), ctypes.byref(shp), 0.5, P(16), P(16), 64, None, P(16), 16,
                             None)
    assert rc == sdl.SDL_ERR_WORKSPACE
    rc = lib.sdl_select_mask(P(16), ctypes.byref(shp), 1.5, P(16), P(16), 64, None, P(16),
                             1 << 20, None)
    assert rc == sdl.SDL_ERR_INVALID_ARG


def test_zero_strides_refused_on_axes_with_more_than_one_index():
    """A broadcast view (stride 0 along tokens, heads or batch) would make distinct
    rows alias one address; every call taking Q/K/V/O refuses it before any launch."""
    import torch
    lib = sdl.lib()
    P = ctypes.c_void_p
    q = torch.zeros(2, 512, 4, 64, dtype=torch.bfloat16)
    k1 = torch.zeros(2, 512, 1, 64, dtype=torch.bfloat16)
    k = k1.expand(2, 512, 4, 64)          # stride 0 along the 4 KV heads
    assert k.stride(2) == 0
    shp = sdl.make_shape(q, k, 64)
    assert shp.k_strides[2] == 0
    rc = lib.sdl_dense_attn(P(16), P(16), P(16), ctypes.byref(shp), 0.0, P(16), None, None)
    assert rc == sdl.SDL_ERR_INVALID_ARG
    rc = lib.sdl_sparse_attn(P(16), P(16), P(16), ctypes.byref(shp), P(16), P(16), 0.0, P(16),
                             None, None)
    assert rc == sdl.SDL_ERR_INVALID_ARG
    # stride 0 along tokens of V, and along the batch of O
    for field, axis in (("v_strides", 1), ("o_strides", 0)):
        bad = sdl.make_shape(q, k1.expand(2, 512, 4, 64).contiguous(), 64)
        getattr(bad, field)[axis] = 0
        rc = lib.sdl_dense_attn(P(16), P(16), P(16), ctypes.byref(bad), 0.0, P(16), None, None)
        assert rc == sdl.SDL_ERR_INVALID_ARG, field
    # an axis of one index may carry any stride: the stride check passes and the
    # call stops at the next host check (no workspace), never reaching a launch
    one = sdl.make_shape(q[:1], k1[:1].expand(1, 512, 4, 64).contiguous(), 64)
    one.q_strides[0] = 0
    rc = lib.sdl_block_scores(P(16), P(16), ctypes.byref(one), 0.0, P(16), None, 0, None)
    assert rc == sdl.SDL_ERR_WORKSPACE
    rc = lib.sdl_block_scores(P(16), P(16), ctypes.byref(shp), 0.0, P(16), None, 0, None)
    assert rc == sdl.SDL_ERR_INVALID_ARG


def test_anchor_step_host_checks():
    """sdl_anchor_step refuses what its header lists before any launch: 128-token
    blocks, a missing plan or order, a short workspace or lists buffer, a
    misaligned lists buffer, a column buffer below the budget."""
    lib = sdl.lib()
    P = ctypes.c_void_p
    shp = _shape(H=4, Hkv=4, L=1024)
    total = sdl.mask_budget(shp, 0.5)
    ws = sdl.lib().sdl_anchor_workspace_bytes(ctypes.byref(shp))
    nl = sdl.lib().sdl_tile_lists_bytes(ctypes.byref(shp))
    assert ws > 0 and nl > 0

    def call(shape=shp, plan=P(256), order=P(256), lists=P(256), lists_bytes=nl, cap=total,
             ws_bytes=ws):
        return lib.sdl_anchor_step(P(256), P(256), ctypes.byref(shape), 0.0, 0.5, P(256),
                                   P(256), P(256), cap, plan, order, lists, lists_bytes, P(256),
                                   ws_bytes, None)

    big = _shape(H=4, Hkv=4, L=1024, block=128)
    assert call(shape=big, ws_bytes=1 << 40) == sdl.SDL_ERR_UNSUPPORTED
    assert call(plan=None) == sdl.SDL_ERR_INVALID_ARG
    assert call(order=None) == sdl.SDL_ERR_INVALID_ARG
    assert call(lists=P(264)) == sdl.SDL_ERR_INVALID_ARG
    assert call(lists_bytes=nl - 1) == sdl.SDL_ERR_WORKSPACE
    assert call(ws_bytes=ws - 1) == sdl.SDL_ERR_WORKSPACE
    assert call(cap=total - 1) == sdl.SDL_ERR_CAPACITY
    rc = lib.sdl_anchor_step(None, P(256), ctypes.byref(shp), 0.0, 0.5, P(256), P(256), P(256),
                             total, P(256), P(256), None, 0, P(256), ws, None)
    assert rc == sdl.SDL_ERR_INVALID_ARG


def test_status_strings():
    lib = sdl.lib()
    for code in range(9):
        assert lib.sdl_status_string(code)
    assert lib.sdl_last_cuda_error() == 0


@pytest.mark.parametrize("B,H,Hkv,L", [(1, 32, 32, 8192), (2, 4, 4, 2112), (1, 28, 4, 16384),
                                       (3, 2, 1, 64)])
def test_tile_lists_size_follows_the_documented_layout(B, H, Hkv, L):
    """Per position of the take order: a record of 8 int32, then a row of 16-bit
    entries, one per 64-token key block, padded to a multiple of 8 entries."""
    lib = sdl.lib()
    shp = _shape(B=B, H=H, Hkv=Hkv, L=L)
    n_items = B * H * -(-L // 128)          # 128-row tiles
    row = -(-(L // 64) // 8) * 8
    want = n_items * 8 * 4 + n_items * row * 2
    assert lib.sdl_tile_lists_bytes(ctypes.byref(shp)) == want
    assert sdl.tile_lists_bytes(B, H, L) == want
    assert want % 16 == 0                   # every row starts 16-byte aligned
    assert lib.sdl_tile_lists_bytes(ctypes.byref(_shape(block=96))) == 0


def test_tile_lists_host_checks():
    lib = sdl.lib()
    P = ctypes.c_void_p
    shp = _shape(H=2, Hkv=2, L=512)
    need = lib.sdl_tile_lists_bytes(ctypes.byref(shp))
    # refused before any CUDA call: null or misaligned buffers, 128-token
    # blocks, too little room
    rc = lib.sdl_tile_lists(P(16), P(16), None, None, ctypes.byref(shp), None, need, None)
    assert rc == sdl.SDL_ERR_INVALID_ARG
    rc = lib.sdl_tile_lists(P(16), P(16), None, None, ctypes.byref(shp), P(24), need, None)
    assert rc == sdl.SDL_ERR_INVALID_ARG
    rc = lib.sdl_tile_lists(None, P(16), None, None, ctypes.byref(shp), P(16), need, None)
    assert rc == sdl.SDL_ERR_INVALID_ARG
    rc = lib.sdl_tile_lists(P(16), P(16), None, None, ctypes.byref(_shape(H=2, Hkv=2, L=512,
                                                                          block=128)),
                            P(16), need, None)
    assert rc == sdl.SDL_ERR_UNSUPPORTED
    rc = lib.sdl_tile_lists(P(16), P(16), None, None, ctypes.byref(shp), P(16), need - 16, None)
    assert rc == sdl.SDL_ERR_WORKSPACE
    # the listed attention call: lists required, bf16 and 64-token blocks only
    rc = lib.sdl_sparse_attn_listed(P(16), P(16), P(16), ctypes.byref(shp), None, 0.0, P(16),
                                    None, None)
    assert rc == sdl.SDL_ERR_INVALID_ARG
    rc = lib.sdl_sparse_attn_listed(P(16), P(16), P(16), ctypes.byref(_shape(H=2, Hkv=2, L=512,
                                                                             dtype=1)),
                                    P(16), 0.0, P(16), None, None)
    assert rc == sdl.SDL_ERR_UNSUPPORTED
    rc = lib.sdl_sparse_attn_listed(P(16), P(16), P(16), ctypes.byref(_shape(H=2, Hkv=2, L=512,
                                                                             block=128)),
                                    P(16), 0.0, P(16), None, None)
    assert rc == sdl.SDL_ERR_UNSUPPORTED


def test_col_scores_workspace_holds_the_block_means_and_row_statistics():
    """The column scores need the block means of Q and K (as the block scores do)
    and a (max, sum) pair per query-block row of every head."""
    lib = sdl.lib()
    for B, H, Hkv, L in ((1, 32, 32, 8192), (2, 28, 4, 16384), (1, 2, 2, 512)):
        shp = _shape(B=B, H=H, Hkv=Hkv, L=L)
        nb = L // 64
        got = lib.sdl_col_scores_workspace_bytes(ctypes.byref(shp))
        assert got >= sdl.scores_workspace_bytes(shp) + 8 * B * H * nb
        assert got % 256 == 0
    assert lib.sdl_col_scores_workspace_bytes(ctypes.byref(_shape(d=96))) == 0


def test_binding_refuses_tile_lists_built_for_a_smaller_shape():
    """The listed attention call takes no buffer size, so the binding checks it on
    the host before the call (CPU tensors: nothing reaches the GPU)."""
    torch = pytest.importorskip("torch")
    B, L, H = 1, 1024, 4
    q = torch.zeros((B, L, H, 128), dtype=torch.bfloat16)
    small = torch.zeros(sdl.tile_lists_bytes(B, H, L // 2), dtype=torch.uint8)
    with pytest.raises(sdl.SdlError) as e:
        sdl.sparse_attn(q, q, q, None, None, 64, out=torch.empty_like(q), lists=small)
    assert e.value.status == sdl.SDL_ERR_WORKSPACE
    # the size counts bytes, whatever the buffer's element type
    as_int32 = torch.zeros(sdl.tile_lists_bytes(B, H, L) // 4 - 1, dtype=torch.int32)
    with pytest.raises(sdl.SdlError):
        sdl.sparse_attn(q, q, q, None, None, 64, out=torch.empty_like(q), lists=as_int32)


def test_binding_refuses_short_or_mistyped_index_buffers():
    """CSR, plan and order buffers are read by the C calls without a size: the
    binding checks their element counts and int32 type first (every call here
    is refused before it reaches the library)."""
    torch = pytest.importorskip("torch")
    B, L, H = 1, 1024, 4
    nb, n_qt = L // 64, L // 128
    q = torch.zeros((B, L, H, 128), dtype=torch.bfloat16)
    rp = torch.zeros(B * H * nb + 1, dtype=torch.int32)
    ci = torch.zeros(8, dtype=torch.int32)
    plan = torch.zeros((B, H, n_qt, 2), dtype=torch.int32)
    order = torch.zeros(B * H * n_qt, dtype=torch.int32)
    cases = [
        dict(row_ptr=rp[:-1], col_idx=ci),
        dict(row_ptr=rp.to(torch.int64), col_idx=ci),
        dict(row_ptr=None, col_idx=ci),
        dict(row_ptr=rp, col_idx=ci.to(torch.int64)),
        dict(row_ptr=rp, col_idx=ci, plan=plan.reshape(-1)[:-1]),
        dict(row_ptr=rp, col_idx=ci, plan=plan, order=order[:-1]),
        dict(row_ptr=rp, col_idx=ci, plan=plan.to(torch.int64), order=order),
    ]
    for kw in cases:
        rpk, cik = kw.pop("row_ptr"), kw.pop("col_idx")
        with pytest.raises(sdl.SdlError) as e:
            sdl.sparse_attn(q, q, q, rpk, cik, 64, out=torch.empty_like(q), **kw)
        assert e.value.status == sdl.SDL_ERR_INVALID_ARG
    with pytest.raises(sdl.SdlError):
        sdl.tile_plan(rp[:-1], ci, B, H, L, 64)
    with pytest.raises(sdl.SdlError):
        sdl.tile_plan(rp, ci, B, H, L, 64, plan=plan.reshape(-1)[:-1])
    with pytest.raises(sdl.SdlError):
        sdl.tile_order(rp, plan.reshape(-1)[:-2], B, H, L, 64)
    with pytest.raises(sdl.SdlError):
        sdl.tile_order(rp, plan, B, H, L, 64, order=order[:-1])
    with pytest.raises(sdl.SdlError):
        sdl.tile_lists(rp, ci, None, order[:-1], B, H, L, 64)
    with pytest.raises(sdl.SdlError):
        sdl.tile_lists(rp[:-1], ci, None, None, B, H, L, 64)


def test_binding_refuses_host_tensors():
    """Every buffer the library reads lives on the device: host tensors of the
    right sizes are refused before the call."""
    torch = pytest.importorskip("torch")
    B, L, H = 1, 512, 2
    nb = L // 64
    q = torch.zeros((B, L, H, 128), dtype=torch.bfloat16)
    rp = torch.zeros(B * H * nb + 1, dtype=torch.int32)
    ci = torch.zeros(8, dtype=torch.int32)
    for call in (lambda: sdl.sparse_attn(q, q, q, rp, ci, 64, out=torch.empty_like(q)),
                 lambda: sdl.dense_attn(q, q, q),
                 lambda: sdl.tile_plan(rp, ci, B, H, L, 64),
                 lambda: sdl.tile_lists(rp, ci, None, None, B, H, L, 64),
                 lambda: sdl.block_scores(q, q, 64),
                 lambda: sdl.select_mask(torch.zeros((B, H, nb, nb)), 0.5, 64, L),
                 lambda: sdl.anchor_refresh(q, q, 64, 0.5),
                 lambda: sdl.col_scores(q, q, 64)):
        with pytest.raises(sdl.SdlError) as e:
            call()
        assert e.value.status == sdl.SDL_ERR_INVALID_ARG


def test_sizing_calls_take_shape_only_probes():
    """Shapes and workspace sizes come from tensors' shapes alone, so the layers
    size their buffers from meta-device probes before any data exists."""
    torch = pytest.importorskip("torch")
    q = torch.empty((1, 8192, 32, 128), dtype=torch.bfloat16, device="meta")
    assert sdl.make_shape(q, q, 64).L == 8192
    assert sdl.anchor_workspace_bytes(q, q, 64) > 0
    assert sdl.col_scores_workspace_bytes(q, q, 64) > 0
    assert sdl.col_budget(q, q, 64, 0.9) == 832
