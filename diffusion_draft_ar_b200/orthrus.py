"""ctypes binding of ``liborthrus.so`` (declared in ``include/orthrus.h``).

Argument marshalling only: every function takes torch tensors that already live
on the GPU, reads their shapes and raw pointers, and calls the C function of the
same name on the current torch stream. All computation happens in the
library's CUDA kernels; there is no fallback, and importing this module fails
loudly when the library has not been built (``python -m
diffusion_draft_ar_b200.build``).
"""
from __future__ import annotations

import ctypes
import os

import torch

VIEW_DIFFUSION = 0
VIEW_VERIFY = 1
VIEWS = {"diffusion": VIEW_DIFFUSION, "verify": VIEW_VERIFY}

FLAG_BAD_PAGE = 0x1
FLAG_BAD_LENGTH = 0x2
FLAG_TIMEOUT = 0x4

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE_CHECK = range(6)

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liborthrus.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built: run `python -m diffusion_draft_ar_b200.build`")

lib = ctypes.CDLL(LIB_PATH)

_i32, _i64, _sz, _vp, _f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float


class AttnParams(ctypes.Structure):
    """Mirror of ``orthrus_attn_params``."""
    _fields_ = [
        ("view", _i32), ("B", _i32), ("Hq", _i32), ("Hkv", _i32), ("D", _i32),
        ("page_size", _i32), ("max_pages_per_seq", _i32), ("num_pages", _i32),
        ("max_block", _i32), ("total_rows", _i32),
        ("q_block", _vp), ("k_cache", _vp), ("v_cache", _vp), ("k_block", _vp), ("v_block", _vp),
        ("prefix_lens", _vp), ("cu_block", _vp), ("page_table", _vp),
        ("softmax_scale", _f32), ("kv_split_tokens", _i32), ("max_ctas", _i32),
        ("out", _vp), ("workspace", _vp), ("workspace_bytes", _sz), ("error_flag", _vp),
    ]


class AttnPlan(ctypes.Structure):
    """Mirror of ``orthrus_attn_plan``."""
    _fields_ = [
        ("schedule", _i32), ("grid", _i32), ("partial_slots", _i32), ("kernels", _i32),
        ("walks_chunks", _i32), ("chunk_tiles", _i32), ("workspace_bytes", _sz),
    ]


SCHEDULES = {0: "balanced", 1: "fixed_chunks", 2: "proportional"}

lib.orthrus_block_attn_workspace_size.restype = _sz
lib.orthrus_block_attn_workspace_size.argtypes = [ctypes.POINTER(AttnParams)]
lib.orthrus_block_attn_plan.restype = _i32
lib.orthrus_block_attn_plan.argtypes = [ctypes.POINTER(AttnParams), _i32, ctypes.POINTER(AttnPlan)]
lib.orthrus_block_attn_kernel_count.restype = _i32
lib.orthrus_block_attn_kernel_count.argtypes = [ctypes.POINTER(AttnParams)]
lib.orthrus_block_attn.restype = _i32
lib.orthrus_block_attn.argtypes = [ctypes.POINTER(AttnParams), _vp]
lib.orthrus_block_attn_verify_write.restype = _i32
lib.orthrus_block_attn_verify_write.argtypes = [ctypes.POINTER(AttnParams), _vp]
lib.orthrus_consensus_workspace_size.restype = _sz
lib.orthrus_consensus_workspace_size.argtypes = [_i32, _i32, _i32]
lib.orthrus_consensus.restype = _i32
lib.orthrus_consensus.argtypes = [_vp, _i64, _i32, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _vp, _sz, _vp]
lib.orthrus_consensus_commit.restype = _i32
lib.orthrus_consensus_commit.argtypes = [_vp, _i64, _i32, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _vp,
                                         _vp, _sz, _vp]
lib.orthrus_kv_append.restype = _i32
lib.orthrus_kv_append.argtypes = [_vp, _vp, _vp, _i32, _vp, _vp, _i32, _vp, _i32, _i32, _vp, _vp,
                                  _i32, _i32, _i32, _i32, _vp, _vp]
lib.orthrus_lm_head_workspace_size.restype = _sz
lib.orthrus_lm_head_workspace_size.argtypes = [_i32]
lib.orthrus_lm_head_consensus.restype = _i32
lib.orthrus_lm_head_consensus.argtypes = [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _i32, _i32, _vp, _vp,
                                          _vp, _vp, _vp, _sz, _vp, _vp]
lib.orthrus_consensus_sampled.restype = _i32
lib.orthrus_consensus_sampled.argtypes = [_vp, _i64, _i32, _vp, _vp, _i32, _i32, _f32,
                                          ctypes.c_uint64, ctypes.c_uint64, _vp, _vp, _vp, _vp,
                                          _vp, _sz, _vp]
lib.orthrus_consensus_noalloc.restype = _i32
lib.orthrus_consensus_noalloc.argtypes = [_vp, _i64, _i32, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _vp]
lib.orthrus_status_string.restype = ctypes.c_char_p
lib.orthrus_status_string.argtypes = [_i32]
lib.orthrus_last_error.restype = ctypes.c_char_p
lib.orthrus_last_error.argtypes = []
lib.orthrus_abi_version.restype = _i32
lib.orthrus_abi_version.argtypes = []
lib.orthrus_status_from_flags.restype = _i32
lib.orthrus_status_from_flags.argtypes = [_i32]


class OrthrusError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = lib.orthrus_last_error().decode()
        super().__init__(f"{where}: {lib.orthrus_status_string(status).decode()} ({detail})")


def _check(status: int, where: str):
    if status != OK:
        raise OrthrusError(status, where)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int | None = None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")


def attn_params(view, q_block, k_cache, v_cache, k_block, v_block, prefix_lens, cu_block,
                page_table, out, max_block: int, workspace=None, softmax_scale: float = 0.0,
                kv_split_tokens: int = 0, max_ctas: int = 0, error_flag=None) -> AttnParams:
    """Fill an ``orthrus_attn_params`` from tensors (shapes read, nothing computed)."""
    v = VIEWS[view] if isinstance(view, str) else int(view)
    _need(q_block, "q_block", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(k_block, "k_block", torch.bfloat16, 3)
    _need(v_block, "v_block", torch.bfloat16, 3)
    _need(prefix_lens, "prefix_lens", torch.int32, 1)
    _need(page_table, "page_table", torch.int32, 2)
    _need(out, "out", torch.bfloat16, 3)
    if cu_block is not None:
        _need(cu_block, "cu_block", torch.int32, 1)
    if error_flag is not None:
        _need(error_flag, "error_flag", torch.int32)
    R, Hq, D = q_block.shape
    num_pages, Hkv, P, _ = k_cache.shape
    p = AttnParams()
    p.view, p.B, p.Hq, p.Hkv, p.D = v, prefix_lens.shape[0], Hq, Hkv, D
    p.page_size, p.max_pages_per_seq, p.num_pages = P, page_table.shape[1], num_pages
    p.max_block, p.total_rows = int(max_block), R
    p.q_block, p.k_cache, p.v_cache = q_block.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr()
    p.k_block, p.v_block = k_block.data_ptr(), v_block.data_ptr()
    p.prefix_lens, p.page_table = prefix_lens.data_ptr(), page_table.data_ptr()
    p.cu_block = cu_block.data_ptr() if cu_block is not None else None
    p.softmax_scale = float(softmax_scale)
    p.kv_split_tokens, p.max_ctas = int(kv_split_tokens), int(max_ctas)
    p.out = out.data_ptr()
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8)
        p.workspace, p.workspace_bytes = workspace.data_ptr(), workspace.numel()
    p.error_flag = error_flag.data_ptr() if error_flag is not None else None
    return p


def block_attn_workspace_size(params: AttnParams) -> int:
    return int(lib.orthrus_block_attn_workspace_size(ctypes.byref(params)))


def block_attn_kernel_count(params: AttnParams) -> int:
    """Kernels one ``orthrus_block_attn`` call with these parameters launches."""
    return int(lib.orthrus_block_attn_kernel_count(ctypes.byref(params)))


def block_attn_plan(params: AttnParams, sm_count: int = 0) -> AttnPlan:
    """``orthrus_block_attn_plan``: the schedule a call with these parameters
    uses on ``sm_count`` SMs (0: the current device's)."""
    plan = AttnPlan()
    _check(lib.orthrus_block_attn_plan(ctypes.byref(params), int(sm_count), ctypes.byref(plan)),
           "orthrus_block_attn_plan")
    return plan


def block_attn(view, q_block, k_cache, v_cache, k_block, v_block, prefix_lens, cu_block,
               page_table, out, workspace, max_block: int, softmax_scale: float = 0.0,
               kv_split_tokens: int = 0, max_ctas: int = 0, error_flag=None, stream=None):
    """``orthrus_block_attn`` on the current stream; ``out`` is written in place."""
    p = attn_params(view, q_block, k_cache, v_cache, k_block, v_block, prefix_lens, cu_block,
                    page_table, out, max_block, workspace, softmax_scale, kv_split_tokens,
                    max_ctas, error_flag)
    _check(lib.orthrus_block_attn(ctypes.byref(p), _stream(stream)), "orthrus_block_attn")
    return out


def block_attn_verify_write(q_block, k_cache, v_cache, k_block, v_block, prefix_lens, cu_block,
                            page_table, out, workspace, max_block: int, softmax_scale: float = 0.0,
                            kv_split_tokens: int = 0, max_ctas: int = 0, error_flag=None,
                            stream=None):
    """``orthrus_block_attn_verify_write``: VERIFY attention that also stores every
    block row's K/V past each prefix (k_cache / v_cache written in place; the
    lengths are left for ``consensus_commit``)."""
    p = attn_params("verify", q_block, k_cache, v_cache, k_block, v_block, prefix_lens,
                    cu_block, page_table, out, max_block, workspace, softmax_scale,
                    kv_split_tokens, max_ctas, error_flag)
    _check(lib.orthrus_block_attn_verify_write(ctypes.byref(p), _stream(stream)),
           "orthrus_block_attn_verify_write")
    return out


def consensus_workspace_size(B: int, max_block: int, V: int) -> int:
    return int(lib.orthrus_consensus_workspace_size(B, max_block, V))


def consensus(verify_logits, draft_tokens, cu_block, B: int, max_block: int, accept_len,
              next_token, workspace, row_argmax=None, stream=None, prefix_lens=None):
    """``orthrus_consensus``: writes accept_len, next_token (and row_argmax) in place.
    With ``prefix_lens`` it is ``orthrus_consensus_commit``: the lengths also
    advance by the accepted counts (after ``block_attn_verify_write``)."""
    if not verify_logits.is_cuda or verify_logits.dtype != torch.float32 or verify_logits.dim() != 2:
        raise ValueError("verify_logits must be a 2-D CUDA float32 tensor")
    if verify_logits.stride(1) != 1:
        raise ValueError("verify_logits rows must be contiguous")
    _need(draft_tokens, "draft_tokens", torch.int32, 1)
    _need(accept_len, "accept_len", torch.int32, 1)
    _need(next_token, "next_token", torch.int32, 1)
    _need(workspace, "workspace", torch.uint8)
    if cu_block is not None:
        _need(cu_block, "cu_block", torch.int32, 1)
    if row_argmax is not None:
        _need(row_argmax, "row_argmax", torch.int32, 1)
    V = verify_logits.shape[1]
    if prefix_lens is not None:
        _need(prefix_lens, "prefix_lens", torch.int32, 1)
        st = lib.orthrus_consensus_commit(_ptr(verify_logits), verify_logits.stride(0), V,
                                          _ptr(draft_tokens), _ptr(cu_block), int(B),
                                          int(max_block), _ptr(accept_len), _ptr(next_token),
                                          _ptr(row_argmax), _ptr(prefix_lens), _ptr(workspace),
                                          workspace.numel(), _stream(stream))
        _check(st, "orthrus_consensus_commit")
        return
    st = lib.orthrus_consensus(_ptr(verify_logits), verify_logits.stride(0), V, _ptr(draft_tokens),
                               _ptr(cu_block), int(B), int(max_block), _ptr(accept_len),
                               _ptr(next_token), _ptr(row_argmax), _ptr(workspace),
                               workspace.numel(), _stream(stream))
    _check(st, "orthrus_consensus")


def consensus_sampled(verify_logits, draft_tokens, cu_block, B: int, max_block: int,
                      temperature: float, seed: int, offset: int, accept_len, next_token,
                      workspace, row_token=None, prefix_lens=None, stream=None):
    """``orthrus_consensus_sampled``: consensus at temperature > 0 (Gumbel-max
    sample of softmax(logits / T) from Philox4x32-10 noise); writes accept_len,
    next_token (and row_token, and advances prefix_lens when given) in place."""
    if not verify_logits.is_cuda or verify_logits.dtype != torch.float32 or verify_logits.dim() != 2:
        raise ValueError("verify_logits must be a 2-D CUDA float32 tensor")
    if verify_logits.stride(1) != 1:
        raise ValueError("verify_logits rows must be contiguous")
    _need(draft_tokens, "draft_tokens", torch.int32, 1)
    _need(accept_len, "accept_len", torch.int32, 1)
    _need(next_token, "next_token", torch.int32, 1)
    _need(workspace, "workspace", torch.uint8)
    for name, t in (("cu_block", cu_block), ("row_token", row_token),
                    ("prefix_lens", prefix_lens)):
        if t is not None:
            _need(t, name, torch.int32, 1)
    st = lib.orthrus_consensus_sampled(_ptr(verify_logits), verify_logits.stride(0),
                                       verify_logits.shape[1], _ptr(draft_tokens), _ptr(cu_block),
                                       int(B), int(max_block), float(temperature),
                                       int(seed) & (2 ** 64 - 1), int(offset) & (2 ** 64 - 1),
                                       _ptr(accept_len), _ptr(next_token), _ptr(row_token),
                                       _ptr(prefix_lens), _ptr(workspace), workspace.numel(),
                                       _stream(stream))
    _check(st, "orthrus_consensus_sampled")


def consensus_noalloc(verify_logits, draft_tokens, cu_block, B: int, max_block: int, accept_len,
                      next_token, row_argmax=None, stream=None):
    """``orthrus_consensus_noalloc``: consensus for callers that cannot hand the
    library a device workspace (the scratch is a fixed array inside the library;
    see the header for its size limit and the rule on overlapping calls)."""
    if not verify_logits.is_cuda or verify_logits.dtype != torch.float32 or verify_logits.dim() != 2:
        raise ValueError("verify_logits must be a 2-D CUDA float32 tensor")
    if verify_logits.stride(1) != 1:
        raise ValueError("verify_logits rows must be contiguous")
    _need(draft_tokens, "draft_tokens", torch.int32, 1)
    _need(accept_len, "accept_len", torch.int32, 1)
    _need(next_token, "next_token", torch.int32, 1)
    if cu_block is not None:
        _need(cu_block, "cu_block", torch.int32, 1)
    if row_argmax is not None:
        _need(row_argmax, "row_argmax", torch.int32, 1)
    st = lib.orthrus_consensus_noalloc(_ptr(verify_logits), verify_logits.stride(0),
                                       verify_logits.shape[1], _ptr(draft_tokens), _ptr(cu_block),
                                       int(B), int(max_block), _ptr(accept_len), _ptr(next_token),
                                       _ptr(row_argmax), _stream(stream))
    _check(st, "orthrus_consensus_noalloc")


def lm_head_workspace_size(total_rows: int) -> int:
    return int(lib.orthrus_lm_head_workspace_size(int(total_rows)))


def lm_head_consensus(hidden, w_head, draft_tokens, cu_block, B: int, max_block: int, accept_len,
                      next_token, workspace, row_argmax=None, prefix_lens=None, error_flag=None,
                      stream=None):
    """``orthrus_lm_head_consensus``: greedy tokens of ``hidden @ w_head.T`` (never
    materialised) and the consensus outputs, written in place."""
    _need(hidden, "hidden", torch.bfloat16, 2)
    _need(w_head, "w_head", torch.bfloat16, 2)
    if hidden.shape[1] != w_head.shape[1]:
        raise ValueError("hidden and w_head must share d_model")
    _need(draft_tokens, "draft_tokens", torch.int32, 1)
    _need(accept_len, "accept_len", torch.int32, 1)
    _need(next_token, "next_token", torch.int32, 1)
    _need(workspace, "workspace", torch.uint8)
    for name, t in (("cu_block", cu_block), ("row_argmax", row_argmax),
                    ("prefix_lens", prefix_lens), ("error_flag", error_flag)):
        if t is not None:
            _need(t, name, torch.int32)
    st = lib.orthrus_lm_head_consensus(_ptr(hidden), _ptr(w_head), hidden.shape[1],
                                       w_head.shape[0], hidden.shape[0], _ptr(draft_tokens),
                                       _ptr(cu_block), int(B), int(max_block), _ptr(accept_len),
                                       _ptr(next_token), _ptr(row_argmax), _ptr(prefix_lens),
                                       _ptr(workspace), workspace.numel(), _ptr(error_flag),
                                       _stream(stream))
    _check(st, "orthrus_lm_head_consensus")


def kv_append(k_block, v_block, cu_block, max_block: int, accept_len, prefix_lens, page_table,
              k_cache, v_cache, update_lens: bool = True, error_flag=None, stream=None):
    """``orthrus_kv_append``: scatters accepted rows into the caches in place."""
    _need(k_block, "k_block", torch.bfloat16, 3)
    _need(v_block, "v_block", torch.bfloat16, 3)
    _need(accept_len, "accept_len", torch.int32, 1)
    _need(prefix_lens, "prefix_lens", torch.int32, 1)
    _need(page_table, "page_table", torch.int32, 2)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    if cu_block is not None:
        _need(cu_block, "cu_block", torch.int32, 1)
    if error_flag is not None:
        _need(error_flag, "error_flag", torch.int32)
    num_pages, Hkv, P, D = k_cache.shape
    st = lib.orthrus_kv_append(_ptr(k_block), _ptr(v_block), _ptr(cu_block), int(max_block),
                               _ptr(accept_len), _ptr(prefix_lens), int(bool(update_lens)),
                               _ptr(page_table), page_table.shape[1], num_pages, _ptr(k_cache),
                               _ptr(v_cache), prefix_lens.shape[0], Hkv, D, P, _ptr(error_flag),
                               _stream(stream))
    _check(st, "orthrus_kv_append")


def abi_version() -> int:
    return int(lib.orthrus_abi_version())
