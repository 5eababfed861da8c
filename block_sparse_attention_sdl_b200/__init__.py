"""Python binding of libsdl: block-sparse attention for diffusion-LLM denoising on B200.

Argument marshalling only.  Every step runs in the CUDA kernels of ``libsdl.so``
(built in-tree by :mod:`block_sparse_attention_sdl_b200.build`); PyTorch supplies
device memory and streams.  There is no CPU fallback: importing this package on a
machine without the built library raises.

Tensors are laid out [B, L, heads, d] with the head dimension contiguous (any
strides on the other axes).  The calls mirror ``include/sdl.h``:

* :func:`block_scores`  pooled block scores with a row softmax (anchor steps)
* :func:`select_mask`   head-adaptive global top-k block mask as CSR (anchor steps)
* :func:`sparse_attn`   block-sparse attention over the kept blocks (every step)
* :func:`dense_attn`    dense bidirectional attention (the baseline)
"""
from __future__ import annotations

import ctypes
import functools
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsdl.so")

SDL_OK, SDL_ERR_INVALID_ARG, SDL_ERR_UNSUPPORTED, SDL_ERR_CAPACITY = 0, 1, 2, 3
SDL_ERR_WORKSPACE, SDL_ERR_CUDA, SDL_ERR_TIMEOUT, SDL_ERR_BAD_MASK = 4, 5, 6, 7
SDL_ERR_OVERLAP = 8
SDL_BF16, SDL_FP32 = 0, 1

EXPORTS = ("sdl_mask_budget", "sdl_scores_workspace_bytes", "sdl_select_workspace_bytes",
           "sdl_mask_budget_scoped", "sdl_select_workspace_bytes_scoped", "sdl_select_mask_scoped",
           "sdl_block_scores", "sdl_select_mask", "sdl_select_mask_noalloc", "sdl_sparse_attn",
           "sdl_tile_plan", "sdl_sparse_attn_planned", "sdl_tile_order",
           "sdl_sparse_attn_scheduled", "sdl_tile_lists_bytes", "sdl_tile_lists",
           "sdl_sparse_attn_listed", "sdl_dense_attn",
           "sdl_anchor_workspace_bytes", "sdl_anchor_refresh", "sdl_anchor_step",
           "sdl_col_budget", "sdl_col_scores_workspace_bytes", "sdl_col_scores",
           "sdl_col_select", "sdl_col_gather", "sdl_col_sparse_attn",
           "sdl_select_shard_workspace_bytes", "sdl_select_shard_hist",
           "sdl_select_shard_capacity", "sdl_select_shard_pass", "sdl_select_shard_count",
           "sdl_select_shard_finish",
           "sdl_wait_selfcheck",
           "sdl_last_device_status", "sdl_last_device_detail", "sdl_last_cuda_error",
           "sdl_status_string")
SDL_SELECT_PASSES = 3


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("H_kv", ctypes.c_int32),
                ("L", ctypes.c_int32), ("d", ctypes.c_int32), ("block", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("q_strides", ctypes.c_int64 * 3), ("k_strides", ctypes.c_int64 * 3),
                ("v_strides", ctypes.c_int64 * 3), ("o_strides", ctypes.c_int64 * 3)]


class SdlError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = _lib().sdl_status_string(status).decode()
        if status == SDL_ERR_CUDA:
            msg += f" (cudaError {_lib().sdl_last_cuda_error()})"
        super().__init__(f"{what}: {msg}")


_L = None


def _lib():
    global _L
    if _L is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m block_sparse_attention_sdl_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, SZ, D, F = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_double,
                            ctypes.c_float)
        SP = ctypes.POINTER(Shape)
        L.sdl_mask_budget.argtypes = [SP, D]
        L.sdl_mask_budget.restype = I64
        L.sdl_scores_workspace_bytes.argtypes = [SP]
        L.sdl_scores_workspace_bytes.restype = SZ
        L.sdl_select_workspace_bytes.argtypes = [SP]
        L.sdl_select_workspace_bytes.restype = SZ
        L.sdl_mask_budget_scoped.argtypes = [SP, D, ctypes.c_int]
        L.sdl_mask_budget_scoped.restype = I64
        L.sdl_select_workspace_bytes_scoped.argtypes = [SP, ctypes.c_int]
        L.sdl_select_workspace_bytes_scoped.restype = SZ
        L.sdl_select_mask_scoped.argtypes = [P, SP, D, ctypes.c_int, P, P, I64, P, P, SZ, P]
        L.sdl_block_scores.argtypes = [P, P, SP, F, P, P, SZ, P]
        L.sdl_select_mask.argtypes = [P, SP, D, P, P, I64, P, P, SZ, P]
        L.sdl_sparse_attn.argtypes = [P, P, P, SP, P, P, F, P, P, P]
        L.sdl_tile_plan.argtypes = [P, P, SP, P, P]
        L.sdl_sparse_attn_planned.argtypes = [P, P, P, SP, P, P, P, F, P, P, P]
        L.sdl_tile_order.argtypes = [P, P, SP, P, P]
        L.sdl_sparse_attn_scheduled.argtypes = [P, P, P, SP, P, P, P, P, F, P, P, P]
        L.sdl_tile_lists_bytes.argtypes = [SP]
        L.sdl_tile_lists_bytes.restype = ctypes.c_size_t
        L.sdl_tile_lists.argtypes = [P, P, P, P, SP, P, ctypes.c_size_t, P]
        L.sdl_sparse_attn_listed.argtypes = [P, P, P, SP, P, F, P, P, P]
        L.sdl_dense_attn.argtypes = [P, P, P, SP, F, P, P, P]
        L.sdl_col_budget.argtypes = [SP, D]
        L.sdl_col_budget.restype = I64
        L.sdl_col_scores_workspace_bytes.argtypes = [SP]
        L.sdl_col_scores_workspace_bytes.restype = SZ
        L.sdl_col_scores.argtypes = [P, P, SP, F, P, P, SZ, P]
        L.sdl_col_select.argtypes = [P, SP, D, P, I64, P]
        L.sdl_col_gather.argtypes = [P, P, SP, P, ctypes.c_int32, P, P, P]
        L.sdl_col_sparse_attn.argtypes = [P, P, P, SP, ctypes.c_int32, F, P, P, P]
        L.sdl_anchor_workspace_bytes.argtypes = [SP]
        L.sdl_anchor_workspace_bytes.restype = SZ
        L.sdl_anchor_refresh.argtypes = [P, P, SP, F, D, P, P, P, I64, P, P, SZ, P]
        L.sdl_anchor_step.argtypes = [P, P, SP, F, D, P, P, P, I64, P, P, P, SZ, P, SZ, P]
        L.sdl_select_shard_workspace_bytes.argtypes = [SP]
        L.sdl_select_shard_workspace_bytes.restype = SZ
        L.sdl_select_shard_hist.argtypes = [SP, ctypes.c_int, ctypes.POINTER(SZ),
                                            ctypes.POINTER(SZ)]
        L.sdl_select_shard_capacity.argtypes = [SP, ctypes.c_int32, D]
        L.sdl_select_shard_capacity.restype = I64
        L.sdl_select_shard_pass.argtypes = [P, SP, ctypes.c_int32, D, ctypes.c_int, P, SZ, P]
        L.sdl_select_shard_count.argtypes = [P, SP, ctypes.c_int32, D, P, SZ, P, P]
        L.sdl_select_shard_finish.argtypes = [P, SP, ctypes.c_int32, D, P, P, P, I64, P, P, SZ,
                                              P]
        L.sdl_wait_selfcheck.argtypes = [ctypes.c_uint64, P]
        L.sdl_last_device_status.argtypes = [P]
        L.sdl_last_cuda_error.argtypes = []
        L.sdl_last_device_detail.argtypes = []
        L.sdl_status_string.argtypes = [ctypes.c_int]
        L.sdl_status_string.restype = ctypes.c_char_p
        for f in ("sdl_block_scores", "sdl_select_mask", "sdl_select_mask_scoped",
                  "sdl_anchor_refresh", "sdl_anchor_step", "sdl_col_scores", "sdl_col_select",
                  "sdl_wait_selfcheck",
                  "sdl_col_gather", "sdl_col_sparse_attn",
                  "sdl_select_shard_hist", "sdl_select_shard_pass", "sdl_select_shard_count",
                  "sdl_select_shard_finish",
                  "sdl_sparse_attn", "sdl_tile_plan",
                  "sdl_sparse_attn_planned", "sdl_tile_order", "sdl_sparse_attn_scheduled",
                  "sdl_tile_lists", "sdl_sparse_attn_listed",
                  "sdl_dense_attn",
                  "sdl_last_device_status", "sdl_last_device_detail", "sdl_last_cuda_error"):
            getattr(L, f).restype = ctypes.c_int
        _L = L
    return _L


def lib():
    """The loaded ``libsdl.so`` (ctypes handle)."""
    return _lib()


def _check(rc: int, what: str):
    if rc != SDL_OK:
        raise SdlError(rc, what)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return SDL_BF16
    if t.dtype == torch.float32:
        return SDL_FP32
    raise TypeError(f"libsdl takes bf16 or fp32 tensors, got {t.dtype}")


def _strides(t):
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("tensors are [B, L, heads, d] with a contiguous head dimension")
    return (t.stride(0), t.stride(1), t.stride(2))


_SHAPES = {}  # built shapes by the tensors' geometry (a step loop repeats a few)


def make_shape(q, k, block: int, v=None, o=None) -> Shape:
    """sdl_shape for Q [B,L,H,d] and K/V [B,L,H_kv,d] tensors (any device: only their
    shapes, dtype and strides are read).  Returns a fresh struct the caller may modify."""
    key = (q.shape, q.stride(), q.dtype, k.shape, k.stride(), k.dtype,
           None if v is None else (v.shape, v.stride()),
           None if o is None else (o.shape, o.stride()), block)
    s = _SHAPES.get(key)
    if s is None:
        B, L, H, d = q.shape
        s = Shape()
        s.B, s.H, s.H_kv, s.L, s.d, s.block = B, H, k.shape[2], L, d, block
        s.dtype = _dtype_code(q)
        s.q_strides[:] = _strides(q)
        s.k_strides[:] = _strides(k)
        s.v_strides[:] = _strides(v if v is not None else k)
        s.o_strides[:] = _strides(o if o is not None else q)
        if len(_SHAPES) >= 64:
            _SHAPES.clear()
        _SHAPES[key] = s
    return Shape.from_buffer_copy(s)


def _stream(stream):
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


SDL_BUDGET_SEQUENCE, SDL_BUDGET_HEAD = 0, 1


def mask_budget(shape: Shape, sparsity: float, per_head: bool = False) -> int:
    """Kept blocks of a call: head-adaptive budget per sequence, or uniform per head."""
    if per_head:
        return int(_lib().sdl_mask_budget_scoped(ctypes.byref(shape), float(sparsity),
                                                 SDL_BUDGET_HEAD))
    return int(_lib().sdl_mask_budget(ctypes.byref(shape), float(sparsity)))


def scores_workspace_bytes(shape: Shape) -> int:
    return int(_lib().sdl_scores_workspace_bytes(ctypes.byref(shape)))


def select_workspace_bytes(shape: Shape, per_head: bool = False) -> int:
    if per_head:
        return int(_lib().sdl_select_workspace_bytes_scoped(ctypes.byref(shape), SDL_BUDGET_HEAD))
    return int(_lib().sdl_select_workspace_bytes(ctypes.byref(shape)))


def _workspace(nbytes, device, ws):
    import torch
    if ws is None:
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
    return ws


def block_scores(q, k, block: int, scale: float = 0.0, scores=None, workspace=None, stream=None):
    """fp32 [B, H, nb, nb] block scores (see ``sdl_block_scores``)."""
    import torch
    s = make_shape(q, k, block)
    nb = s.L // block
    if scores is None:
        scores = torch.empty((s.B, s.H, nb, nb), dtype=torch.float32, device=q.device)
    need = scores_workspace_bytes(s)
    workspace = _workspace(need, q.device, workspace)
    _on_cuda("sdl_block_scores", q, k, scores, workspace)
    _check(_lib().sdl_block_scores(q.data_ptr(), k.data_ptr(), ctypes.byref(s), float(scale),
                                   scores.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                   _stream(stream)), "sdl_block_scores")
    return scores


def select_mask(scores, sparsity: float, block: int, L: int, row_ptr=None, col_idx=None,
                mask=None, want_mask: bool = False, workspace=None, per_head: bool = False,
                stream=None):
    """(row_ptr int32 [B*H*nb+1], col_idx int32 [budget], mask uint8 or None); ``per_head``
    takes a uniform budget per head instead of the head-adaptive one per sequence."""
    import torch
    B, H, nb, _ = scores.shape
    s = Shape()
    s.B, s.H, s.H_kv, s.L, s.d, s.block, s.dtype = B, H, H, L, 64, block, SDL_FP32
    if nb != L // block:
        raise ValueError("scores shape does not match L / block")
    total = mask_budget(s, sparsity, per_head)
    if total < 0:
        raise SdlError(SDL_ERR_INVALID_ARG, "sdl_mask_budget")
    dev = scores.device
    if row_ptr is None:
        row_ptr = torch.empty(B * H * nb + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        col_idx = torch.empty(total, dtype=torch.int32, device=dev)
    if mask is None and want_mask:
        mask = torch.empty((B, H, nb, nb), dtype=torch.uint8, device=dev)
    workspace = _workspace(select_workspace_bytes(s, per_head), dev, workspace)
    mask_ptr = None if mask is None else mask.data_ptr()
    if per_head:
        _on_cuda("sdl_select_mask_scoped", scores, row_ptr, col_idx, workspace, mask)
        _check(_lib().sdl_select_mask_scoped(scores.data_ptr(), ctypes.byref(s), float(sparsity),
                                             SDL_BUDGET_HEAD, row_ptr.data_ptr(),
                                             col_idx.data_ptr(), col_idx.numel(), mask_ptr,
                                             workspace.data_ptr(), workspace.numel(),
                                             _stream(stream)), "sdl_select_mask_scoped")
    else:
        _on_cuda("sdl_select_mask", scores, row_ptr, col_idx, workspace, mask)
        _check(_lib().sdl_select_mask(scores.data_ptr(), ctypes.byref(s), float(sparsity),
                                      row_ptr.data_ptr(), col_idx.data_ptr(), col_idx.numel(),
                                      mask_ptr, workspace.data_ptr(), workspace.numel(),
                                      _stream(stream)), "sdl_select_mask")
    return row_ptr, col_idx, mask


def anchor_workspace_bytes(q, k, block: int) -> int:
    return int(_lib().sdl_anchor_workspace_bytes(ctypes.byref(make_shape(q, k, block))))


def anchor_refresh(q, k, block: int, sparsity: float, scores=None, row_ptr=None, col_idx=None,
                   plan=None, want_plan: bool = True, workspace=None, scale: float = 0.0,
                   stream=None):
    """Block scores, mask selection and (64-token blocks) the tile plan in one launch
    (see ``sdl_anchor_refresh``); returns (scores, row_ptr, col_idx, plan or None)."""
    import torch
    s = make_shape(q, k, block)
    nb = s.L // block
    dev = q.device
    total = mask_budget(s, sparsity)
    if total < 0:
        raise SdlError(SDL_ERR_INVALID_ARG, "sdl_mask_budget")
    if scores is None:
        scores = torch.empty((s.B, s.H, nb, nb), dtype=torch.float32, device=dev)
    if row_ptr is None:
        row_ptr = torch.empty(s.B * s.H * nb + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        col_idx = torch.empty(total, dtype=torch.int32, device=dev)
    if plan is None and want_plan and block == 64:
        plan = torch.empty((s.B, s.H, (nb + 1) // 2, 2), dtype=torch.int32, device=dev)
    workspace = _workspace(anchor_workspace_bytes(q, k, block), dev, workspace)
    _on_cuda("sdl_anchor_refresh", q, k, scores, row_ptr, col_idx, plan, workspace)
    _check(_lib().sdl_anchor_refresh(q.data_ptr(), k.data_ptr(), ctypes.byref(s), float(scale),
                                     float(sparsity), scores.data_ptr(), row_ptr.data_ptr(),
                                     col_idx.data_ptr(), col_idx.numel(),
                                     None if plan is None else plan.data_ptr(),
                                     workspace.data_ptr(), workspace.numel(), _stream(stream)),
           "sdl_anchor_refresh")
    return scores, row_ptr, col_idx, plan


def anchor_step(q, k, block: int, sparsity: float, scores=None, row_ptr=None, col_idx=None,
                plan=None, order=None, lists=None, want_lists: bool = True, workspace=None,
                scale: float = 0.0, stream=None):
    """The whole anchor step in one call (see ``sdl_anchor_step``): block scores, mask,
    tile plan, take order and (``want_lists``) the tile lists; 64-token blocks.
    Returns (scores, row_ptr, col_idx, plan, order, lists or None)."""
    import torch
    s = make_shape(q, k, block)
    nb = s.L // block
    dev = q.device
    n_qt = (nb + 1) // 2
    # buffers the caller did not pass (a layer passes all of them: no host work here)
    if scores is None:
        scores = torch.empty((s.B, s.H, nb, nb), dtype=torch.float32, device=dev)
    if row_ptr is None:
        row_ptr = torch.empty(s.B * s.H * nb + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        total = mask_budget(s, sparsity)
        if total < 0:
            raise SdlError(SDL_ERR_INVALID_ARG, "sdl_mask_budget")
        col_idx = torch.empty(total, dtype=torch.int32, device=dev)
    if plan is None:
        plan = torch.empty((s.B, s.H, n_qt, 2), dtype=torch.int32, device=dev)
    if order is None:
        order = torch.empty(s.B * s.H * n_qt, dtype=torch.int32, device=dev)
    if lists is None and want_lists:
        lists = torch.empty(int(_lib().sdl_tile_lists_bytes(ctypes.byref(s))), dtype=torch.uint8,
                            device=dev)
    if workspace is None:
        workspace = torch.empty(max(int(_lib().sdl_anchor_workspace_bytes(ctypes.byref(s))), 16),
                                dtype=torch.uint8, device=dev)
    _on_cuda("sdl_anchor_step", q, k, scores, row_ptr, col_idx, plan, order, lists, workspace)
    _check(_lib().sdl_anchor_step(q.data_ptr(), k.data_ptr(), ctypes.byref(s), float(scale),
                                  float(sparsity), scores.data_ptr(), row_ptr.data_ptr(),
                                  col_idx.data_ptr(), col_idx.numel(), plan.data_ptr(),
                                  order.data_ptr(), None if lists is None else lists.data_ptr(),
                                  0 if lists is None else lists.numel(), workspace.data_ptr(),
                                  workspace.numel(), _stream(stream)),
           "sdl_anchor_step")
    return scores, row_ptr, col_idx, plan, order, lists


def col_budget(q, k, block: int, sparsity: float) -> int:
    """Columns kept per head (``sdl_col_budget``)."""
    n = int(_lib().sdl_col_budget(ctypes.byref(make_shape(q, k, block)), float(sparsity)))
    if n < 0:
        raise SdlError(SDL_ERR_INVALID_ARG, "sdl_col_budget")
    return n


def col_scores_workspace_bytes(q, k, block: int) -> int:
    return int(_lib().sdl_col_scores_workspace_bytes(ctypes.byref(make_shape(q, k, block))))


def col_scores(q, k, block: int, scale: float = 0.0, out=None, workspace=None, stream=None):
    """fp32 [B, H, L] column scores (see ``sdl_col_scores``)."""
    import torch
    s = make_shape(q, k, block)
    if out is None:
        out = torch.empty((s.B, s.H, s.L), dtype=torch.float32, device=q.device)
    workspace = _workspace(col_scores_workspace_bytes(q, k, block), q.device, workspace)
    _on_cuda("sdl_col_scores", q, k, out, workspace)
    _check(_lib().sdl_col_scores(q.data_ptr(), k.data_ptr(), ctypes.byref(s), float(scale),
                                 out.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                 _stream(stream)), "sdl_col_scores")
    return out


def col_select(col_scores_, q, k, block: int, sparsity: float, cols=None, stream=None):
    """int32 [B, H, Lc]: each head's kept columns, ascending (see ``sdl_col_select``)."""
    import torch
    s = make_shape(q, k, block)
    Lc = col_budget(q, k, block, sparsity)
    if cols is None:
        cols = torch.empty((s.B, s.H, Lc), dtype=torch.int32, device=q.device)
    _on_cuda("sdl_col_select", col_scores_, cols)
    _check(_lib().sdl_col_select(col_scores_.data_ptr(), ctypes.byref(s), float(sparsity),
                                 cols.data_ptr(), cols.numel(), _stream(stream)),
           "sdl_col_select")
    return cols


def col_gather(k, v, cols, q, block: int, k_cols=None, v_cols=None, stream=None):
    """The kept K and V tokens, [B, Lc, H, d] each (see ``sdl_col_gather``)."""
    import torch
    s = make_shape(q, k, block, v=v)
    Lc = cols.shape[2]
    if k_cols is None:
        k_cols = torch.empty((s.B, Lc, s.H, s.d), dtype=k.dtype, device=k.device)
    if v_cols is None:
        v_cols = torch.empty((s.B, Lc, s.H, s.d), dtype=v.dtype, device=v.device)
    _on_cuda("sdl_col_gather", k, v, cols, k_cols, v_cols)
    _check(_lib().sdl_col_gather(k.data_ptr(), v.data_ptr(), ctypes.byref(s), cols.data_ptr(),
                                 int(Lc), k_cols.data_ptr(), v_cols.data_ptr(), _stream(stream)),
           "sdl_col_gather")
    return k_cols, v_cols


def col_sparse_attn(q, k_cols, v_cols, block: int = 64, scale: float = 0.0, out=None,
                    want_lse: bool = False, lse=None, stream=None):
    """Attention of every query token over its head's gathered columns
    (see ``sdl_col_sparse_attn``); returns out, or (out, lse)."""
    import torch
    Lc = k_cols.shape[1]
    s = make_shape(q, q, block, o=out if out is not None else q)
    if out is None:
        out = torch.empty_like(q)
        s.o_strides[:] = _strides(out)
    if lse is None and want_lse:
        lse = torch.empty((s.B, s.H, s.L), dtype=torch.float32, device=q.device)
    _on_cuda("sdl_col_sparse_attn", q, k_cols, v_cols, out, lse)
    _check(_lib().sdl_col_sparse_attn(q.data_ptr(), k_cols.data_ptr(), v_cols.data_ptr(),
                                      ctypes.byref(s), int(Lc), float(scale), out.data_ptr(),
                                      None if lse is None else lse.data_ptr(), _stream(stream)),
           "sdl_col_sparse_attn")
    return (out, lse) if want_lse else out


def _score_shape(scores, block: int, L: int) -> Shape:
    B, H, nb, _ = scores.shape
    if nb != L // block:
        raise ValueError("scores shape does not match L / block")
    s = Shape()
    s.B, s.H, s.H_kv, s.L, s.d, s.block, s.dtype = B, H, H, L, 64, block, SDL_FP32
    return s


def select_shard_workspace_bytes(scores, block: int, L: int) -> int:
    """Workspace bytes of the staged selection for this rank's part of the heads."""
    return int(_lib().sdl_select_shard_workspace_bytes(ctypes.byref(_score_shape(scores, block, L))))


def select_shard_hist(workspace, scores, block: int, L: int, p: int):
    """int32 view of the pass-``p`` histogram inside the workspace (summed over ranks
    in place between passes)."""
    import torch
    off, cnt = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib().sdl_select_shard_hist(ctypes.byref(_score_shape(scores, block, L)), int(p),
                                        ctypes.byref(off), ctypes.byref(cnt)),
           "sdl_select_shard_hist")
    return workspace[off.value: off.value + 4 * cnt.value].view(torch.int32)


def select_shard_capacity(scores, sparsity: float, block: int, L: int, heads_total: int) -> int:
    n = int(_lib().sdl_select_shard_capacity(ctypes.byref(_score_shape(scores, block, L)),
                                             int(heads_total), float(sparsity)))
    if n < 0:
        raise SdlError(SDL_ERR_INVALID_ARG, "sdl_select_shard_capacity")
    return n


def select_shard_pass(scores, sparsity: float, block: int, L: int, heads_total: int, p: int,
                      workspace, stream=None):
    s = _score_shape(scores, block, L)
    _on_cuda("sdl_select_shard_pass", scores, workspace)
    _check(_lib().sdl_select_shard_pass(scores.data_ptr(), ctypes.byref(s), int(heads_total),
                                        float(sparsity), int(p), workspace.data_ptr(),
                                        workspace.numel(), _stream(stream)),
           "sdl_select_shard_pass")


def select_shard_count(scores, sparsity: float, block: int, L: int, heads_total: int,
                       workspace, totals=None, stream=None):
    """int64 [B, 2]: this rank's keys above and equal to the threshold, per sequence."""
    import torch
    s = _score_shape(scores, block, L)
    if totals is None:
        totals = torch.empty((s.B, 2), dtype=torch.int64, device=scores.device)
    _on_cuda("sdl_select_shard_count", scores, workspace, totals)
    _check(_lib().sdl_select_shard_count(scores.data_ptr(), ctypes.byref(s), int(heads_total),
                                         float(sparsity), workspace.data_ptr(),
                                         workspace.numel(), totals.data_ptr(), _stream(stream)),
           "sdl_select_shard_count")
    return totals


def select_shard_finish(scores, sparsity: float, block: int, L: int, heads_total: int,
                        offsets, workspace, row_ptr=None, col_idx=None, mask=None,
                        want_mask: bool = False, stream=None):
    """This rank's CSR (row_ptr, col_idx with ``select_shard_capacity`` room, mask)."""
    import torch
    s = _score_shape(scores, block, L)
    nb = L // block
    dev = scores.device
    if row_ptr is None:
        row_ptr = torch.empty(s.B * s.H * nb + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        col_idx = torch.empty(select_shard_capacity(scores, sparsity, block, L, heads_total),
                              dtype=torch.int32, device=dev)
    if mask is None and want_mask:
        mask = torch.empty((s.B, s.H, nb, nb), dtype=torch.uint8, device=dev)
    if offsets.dtype != torch.int64 or not offsets.is_contiguous():
        raise ValueError("offsets must be a contiguous int64 [B, 2] tensor")
    _on_cuda("sdl_select_shard_finish", scores, offsets, row_ptr, col_idx, mask, workspace)
    _check(_lib().sdl_select_shard_finish(scores.data_ptr(), ctypes.byref(s), int(heads_total),
                                          float(sparsity), offsets.data_ptr(),
                                          row_ptr.data_ptr(), col_idx.data_ptr(),
                                          col_idx.numel(),
                                          None if mask is None else mask.data_ptr(),
                                          workspace.data_ptr(), workspace.numel(),
                                          _stream(stream)), "sdl_select_shard_finish")
    return row_ptr, col_idx, mask


def tile_order(row_ptr, plan, B: int, H: int, L: int, block: int = 64, order=None,
               stream=None):
    """int32 [B*H*ceil(nb/2)]: the plan's tiles, costliest first (see ``sdl_tile_order``)."""
    import torch
    nb = L // block
    s = Shape()
    s.B, s.H, s.H_kv, s.L, s.d, s.block, s.dtype = B, H, H, L, 64, block, SDL_BF16
    n_qt = (nb + 1) // 2
    _need_i32(row_ptr, B * H * nb + 1, "tile_order row_ptr")
    _need_i32(plan, B * H * n_qt * 2, "tile_order plan")
    if order is None:
        order = torch.empty(B * H * n_qt, dtype=torch.int32, device=plan.device)
    _need_i32(order, B * H * n_qt, "tile_order order")
    _on_cuda("tile_order", row_ptr, plan, order)
    _check(_lib().sdl_tile_order(row_ptr.data_ptr(), plan.data_ptr(), ctypes.byref(s),
                                 order.data_ptr(), _stream(stream)), "sdl_tile_order")
    return order


def _on_cuda(what: str, *tensors):
    """Refuses host tensors: the library would hand their addresses to a kernel."""
    for t in tensors:
        if t is not None and not t.is_cuda:
            raise SdlError(SDL_ERR_INVALID_ARG, f"{what}: CUDA tensors required")


def _need_i32(t, n: int, what: str):
    """Host check of an int32 index buffer that the C call reads without a size."""
    import torch
    if t is None or t.dtype != torch.int32 or t.numel() < n:
        raise SdlError(SDL_ERR_INVALID_ARG, f"{what}: int32 with at least {n} elements needed")


@functools.lru_cache(maxsize=256)
def tile_lists_bytes(B: int, H: int, L: int, block: int = 64) -> int:
    """Bytes of the prebuilt tile lists of a shape (see ``sdl_tile_lists_bytes``)."""
    s = Shape()
    s.B, s.H, s.H_kv, s.L, s.d, s.block, s.dtype = B, H, H, L, 64, block, SDL_BF16
    nbytes = int(_lib().sdl_tile_lists_bytes(ctypes.byref(s)))
    if nbytes == 0:
        raise SdlError(SDL_ERR_INVALID_ARG, "sdl_tile_lists_bytes")
    return nbytes


def tile_lists(row_ptr, col_idx, plan, order, B: int, H: int, L: int, block: int = 64,
               lists=None, stream=None):
    """uint8 buffer of the tiles' kept-block lists in take order (see ``sdl_tile_lists``);
    ``plan`` and ``order`` may be None (adjacent pairs, plan order)."""
    import torch
    s = Shape()
    s.B, s.H, s.H_kv, s.L, s.d, s.block, s.dtype = B, H, H, L, 64, block, SDL_BF16
    nb, n_qt = L // block, (L // block + 1) // 2
    _need_i32(row_ptr, B * H * nb + 1, "tile_lists row_ptr")
    if plan is not None:
        _need_i32(plan, B * H * n_qt * 2, "tile_lists plan")
    if order is not None:
        _need_i32(order, B * H * n_qt, "tile_lists order")
    _need_i32(col_idx, 0, "tile_lists col_idx")
    if lists is None:
        lists = torch.empty(tile_lists_bytes(B, H, L, block), dtype=torch.uint8,
                            device=row_ptr.device)
    _on_cuda("tile_lists", row_ptr, col_idx, plan, order, lists)
    _check(_lib().sdl_tile_lists(row_ptr.data_ptr(), col_idx.data_ptr(),
                                 None if plan is None else plan.data_ptr(),
                                 None if order is None else order.data_ptr(), ctypes.byref(s),
                                 lists.data_ptr(), lists.numel() * lists.element_size(),
                                 _stream(stream)),
           "sdl_tile_lists")
    return lists


def tile_plan(row_ptr, col_idx, B: int, H: int, L: int, block: int = 64, plan=None,
              stream=None):
    """int32 [B, H, ceil(nb/2), 2] tile plan for 64-token blocks (see ``sdl_tile_plan``)."""
    import torch
    nb = L // block
    s = Shape()
    s.B, s.H, s.H_kv, s.L, s.d, s.block, s.dtype = B, H, H, L, 64, block, SDL_BF16
    _need_i32(row_ptr, B * H * nb + 1, "tile_plan row_ptr")
    if plan is None:
        plan = torch.empty((B, H, (nb + 1) // 2, 2), dtype=torch.int32, device=row_ptr.device)
    _need_i32(plan, B * H * ((nb + 1) // 2) * 2, "tile_plan plan")
    _need_i32(col_idx, 0, "tile_plan col_idx")
    _on_cuda("tile_plan", row_ptr, col_idx, plan)
    _check(_lib().sdl_tile_plan(row_ptr.data_ptr(), col_idx.data_ptr(), ctypes.byref(s),
                                plan.data_ptr(), _stream(stream)), "sdl_tile_plan")
    return plan


def sparse_attn(q, k, v, row_ptr, col_idx, block: int, scale: float = 0.0, out=None, lse=None,
                want_lse: bool = False, plan=None, order=None, lists=None, stream=None):
    """O like q (and LSE fp32 [B,H,L] when asked) over the kept blocks; ``plan`` is an
    optional tile plan from :func:`tile_plan` (results equal up to fp32 summation order),
    ``order`` the order of taking its tiles from :func:`tile_order` (same bits), ``lists``
    the tiles' prebuilt lists from :func:`tile_lists` (used instead of the CSR, same bits
    as the plan and order they were built from)."""
    import torch
    B, L, H = q.shape[0], q.shape[1], q.shape[2]
    # the C calls read the lists, CSR, plan and order without a size: checked here
    if lists is not None:
        if lists.numel() * lists.element_size() < tile_lists_bytes(B, H, L, block):
            raise SdlError(SDL_ERR_WORKSPACE, "sdl_sparse_attn_listed: lists too small")
    else:
        nb, n_qt = (L // block if block > 0 else 0), (L + 127) // 128
        _need_i32(row_ptr, B * H * nb + 1, "sparse_attn row_ptr")
        _need_i32(col_idx, 0, "sparse_attn col_idx")
        if plan is not None:
            _need_i32(plan, B * H * n_qt * 2, "sparse_attn plan")
        if order is not None:
            _need_i32(order, B * H * n_qt, "sparse_attn order")
    if out is None:
        out = torch.empty_like(q)
    s = make_shape(q, k, block, v, out)
    if lse is None and want_lse:
        lse = torch.empty((s.B, s.H, s.L), dtype=torch.float32, device=q.device)
    _on_cuda("sparse_attn", q, k, v, out, lse, lists, row_ptr, col_idx, plan, order)
    if lists is not None:
        _check(_lib().sdl_sparse_attn_listed(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                             ctypes.byref(s), lists.data_ptr(), float(scale),
                                             out.data_ptr(),
                                             None if lse is None else lse.data_ptr(),
                                             _stream(stream)), "sdl_sparse_attn_listed")
    else:
        lse_p = None if lse is None else lse.data_ptr()
        if plan is not None and order is not None:
            _check(_lib().sdl_sparse_attn_scheduled(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                    ctypes.byref(s), row_ptr.data_ptr(),
                                                    col_idx.data_ptr(), plan.data_ptr(),
                                                    order.data_ptr(), float(scale),
                                                    out.data_ptr(), lse_p, _stream(stream)),
                   "sdl_sparse_attn_scheduled")
        elif plan is None:
            _check(_lib().sdl_sparse_attn(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                          ctypes.byref(s), row_ptr.data_ptr(),
                                          col_idx.data_ptr(), float(scale), out.data_ptr(),
                                          lse_p, _stream(stream)), "sdl_sparse_attn")
        else:
            _check(_lib().sdl_sparse_attn_planned(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                  ctypes.byref(s), row_ptr.data_ptr(),
                                                  col_idx.data_ptr(), plan.data_ptr(),
                                                  float(scale), out.data_ptr(), lse_p,
                                                  _stream(stream)), "sdl_sparse_attn_planned")
    return (out, lse) if want_lse or lse is not None else out


def dense_attn(q, k, v, block: int = 64, scale: float = 0.0, out=None, lse=None,
               want_lse: bool = False, stream=None):
    """Dense bidirectional attention (the baseline)."""
    import torch
    if out is None:
        out = torch.empty_like(q)
    s = make_shape(q, k, block, v, out)
    if lse is None and want_lse:
        lse = torch.empty((s.B, s.H, s.L), dtype=torch.float32, device=q.device)
    _on_cuda("sdl_dense_attn", q, k, v, out, lse)
    _check(_lib().sdl_dense_attn(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(s),
                                 float(scale), out.data_ptr(),
                                 None if lse is None else lse.data_ptr(), _stream(stream)),
           "sdl_dense_attn")
    return (out, lse) if want_lse or lse is not None else out


def wait_selfcheck(limit_ns: int = 1_000_000, stream=None):
    """Runs the bounded-wait self-check (see ``sdl_wait_selfcheck``); the next
    ``last_device_status`` reports SDL_ERR_TIMEOUT."""
    _check(_lib().sdl_wait_selfcheck(int(limit_ns), _stream(stream)), "sdl_wait_selfcheck")


def last_device_status(stream=None) -> int:
    """Synchronizes the stream and returns (and clears) the kernels' status code."""
    return int(_lib().sdl_last_device_status(_stream(stream)))


BAD_MASK_SITES = {1: "tile plan entry", 2: "CSR entry", 3: "tile-lists record",
                  4: "tile-lists record rows", 5: "tile-lists entry",
                  6: "take-order entry (attention)", 7: "take-order entry (tile lists)",
                  8: "CSR entry (fp32 kernel)"}


def last_device_detail():
    """(site name, offending value) of the bad-mask report behind the last
    :func:`last_device_status` of this thread, or None (``sdl_last_device_detail``)."""
    d = int(_lib().sdl_last_device_detail())
    if d == 0:
        return None
    return BAD_MASK_SITES.get(d >> 24, f"site {d >> 24}"), d & 0xFFFFFF
