"""Thin ctypes binding of the C ABI in ``include/sgqa.h``.

Argument marshalling only: every step of the path runs in ``libsgqa.so``.
Functions take torch tensors (device memory, C-contiguous, in the layouts the
header states) and the current torch CUDA stream.  Errors raise
``SgqaError`` with the library's message.  There is no fallback: if the
library cannot be loaded, importing this module raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsgqa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m sparse_long_context_sgqa_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

STATUS = {0: "SGQA_OK", 1: "SGQA_ERR_INVALID_ARGUMENT", 2: "SGQA_ERR_UNSUPPORTED",
          3: "SGQA_ERR_WORKSPACE", 4: "SGQA_ERR_CUDA", 5: "SGQA_ERR_TIMEOUT", 6: "SGQA_ERR_DEVICE"}

EXPORTED = ["sgqa_workspace_size", "sgqa_merge_blocks", "sgqa_index_topk", "sgqa_sparse_attn",
            "sgqa_sparse_attn_gated", "sgqa_forward", "sgqa_forward_gated", "sgqa_sparse_attn_paged",
            "sgqa_sparse_attn_noalloc",
            "sgqa_set_wait_limit_ns", "sgqa_check", "sgqa_last_error", "sgqa_version", "sgqa_launch_count"]


class SgqaError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


class _Params(ctypes.Structure):
    _fields_ = [("num_kv_groups", ctypes.c_int32), ("heads_per_group", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("idx_heads", ctypes.c_int32),
                ("idx_dim", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("merge_in_f32", ctypes.c_int32),
                ("scale", ctypes.c_float)]


@dataclasses.dataclass
class Params:
    num_kv_groups: int = 4
    heads_per_group: int = 16
    head_dim: int = 192
    idx_heads: int = 8
    idx_dim: int = 64
    block_size: int = 8
    topk: int = 512
    merge_in_f32: int = 0
    scale: float = 0.0

    def c(self) -> _Params:
        return _Params(*dataclasses.astuple(self))


_vp, _i64, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
_P = ctypes.POINTER(_Params)
_lib.sgqa_workspace_size.argtypes = [_P, _i64, _i64, _i64, ctypes.POINTER(_sz)]
_lib.sgqa_merge_blocks.argtypes = [_P, _i64, _i64, _vp, _vp, _i64, _i64, _vp, _vp, _vp]
_lib.sgqa_index_topk.argtypes = [_P, _i64, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.sgqa_sparse_attn.argtypes = [_P, _i64, _i64, _i64, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp,
                                  _vp, _sz, _vp]
_lib.sgqa_sparse_attn_gated.argtypes = [_P, _i64, _i64, _i64, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp,
                                        _vp, _sz, _vp]
_lib.sgqa_forward.argtypes = [_P, _i64, _i64, _i64, _vp, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp,
                              _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.sgqa_forward_gated.argtypes = [_P, _i64, _i64, _i64, _vp, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp,
                                    _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.sgqa_sparse_attn_paged.argtypes = [_P, _i64, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _i64, _i64, _vp, _vp, _vp,
                                        _vp, _vp, _sz, _vp]
_lib.sgqa_sparse_attn_noalloc.argtypes = [_P, _i64, _i64, _i64, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.sgqa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
_lib.sgqa_check.argtypes = [_vp]
_lib.sgqa_last_error.restype = ctypes.c_char_p
_lib.sgqa_version.restype = ctypes.c_char_p
_lib.sgqa_launch_count.restype = ctypes.c_uint64
for _f in EXPORTED[:-3]:
    getattr(_lib, _f).restype = ctypes.c_int


def _ok(code):
    if code != 0:
        raise SgqaError(code, _lib.sgqa_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def version() -> str:
    return _lib.sgqa_version().decode()


def launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(_lib.sgqa_launch_count())


def sgqa_workspace_size(p: Params, num_seqs: int, nq: int, max_ctx: int) -> int:
    out = _sz(0)
    _ok(_lib.sgqa_workspace_size(ctypes.byref(p.c()), num_seqs, nq, max_ctx, ctypes.byref(out)))
    return out.value


def alloc_workspace(p: Params, num_seqs: int, nq: int, max_ctx: int, device) -> torch.Tensor:
    n = sgqa_workspace_size(p, num_seqs, nq, max_ctx)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def sgqa_merge_blocks(p: Params, num_seqs, cache_cap, proxy_k, comp_logits, blk_begin, blk_end,
                      merged_f32, store, stream=None):
    _ok(_lib.sgqa_merge_blocks(ctypes.byref(p.c()), num_seqs, cache_cap, _ptr(proxy_k), _ptr(comp_logits),
                               blk_begin, blk_end, _ptr(merged_f32), _ptr(store), _stream(stream)))


def sgqa_index_topk(p: Params, num_seqs, q_pos0, nq, idx_q, idx_w, cache_cap, store, sel, sel_count,
                    workspace, stream=None):
    _ok(_lib.sgqa_index_topk(ctypes.byref(p.c()), num_seqs, q_pos0, nq, _ptr(idx_q), _ptr(idx_w), cache_cap,
                             _ptr(store), _ptr(sel), _ptr(sel_count), _ptr(workspace),
                             workspace.numel() if workspace is not None else 0, _stream(stream)))


def sgqa_sparse_attn(p: Params, num_seqs, q_pos0, nq, q, cache_cap, cache_len, k_cache, v_cache, sel,
                     sel_count, out, workspace, stream=None):
    _ok(_lib.sgqa_sparse_attn(ctypes.byref(p.c()), num_seqs, q_pos0, nq, _ptr(q), cache_cap, cache_len,
                              _ptr(k_cache), _ptr(v_cache), _ptr(sel), _ptr(sel_count), _ptr(out),
                              _ptr(workspace), workspace.numel() if workspace is not None else 0,
                              _stream(stream)))


def sgqa_sparse_attn_gated(p: Params, num_seqs, q_pos0, nq, q, cache_cap, cache_len, k_cache, v_cache, sel,
                           sel_count, gate, out, workspace, stream=None):
    """sgqa_sparse_attn with the head-wise sigmoid output gate (gate: [S, nq, G*Hg] bf16 logits)."""
    _ok(_lib.sgqa_sparse_attn_gated(ctypes.byref(p.c()), num_seqs, q_pos0, nq, _ptr(q), cache_cap, cache_len,
                                    _ptr(k_cache), _ptr(v_cache), _ptr(sel), _ptr(sel_count), _ptr(gate),
                                    _ptr(out), _ptr(workspace), workspace.numel() if workspace is not None else 0,
                                    _stream(stream)))


def sgqa_forward_gated(p: Params, num_seqs, q_pos0, nq, q, idx_q, idx_w, cache_cap, cache_len, proxy_k,
                       comp_logits, k_cache, v_cache, merged_f32, store, sel, sel_count, gate, out, workspace,
                       stream=None):
    """sgqa_forward with the head-wise sigmoid output gate (gate: [S, nq, G*Hg] bf16 logits)."""
    _ok(_lib.sgqa_forward_gated(ctypes.byref(p.c()), num_seqs, q_pos0, nq, _ptr(q), _ptr(idx_q), _ptr(idx_w),
                                cache_cap, cache_len, _ptr(proxy_k), _ptr(comp_logits), _ptr(k_cache),
                                _ptr(v_cache), _ptr(merged_f32), _ptr(store), _ptr(sel), _ptr(sel_count),
                                _ptr(gate), _ptr(out), _ptr(workspace),
                                workspace.numel() if workspace is not None else 0, _stream(stream)))


def sgqa_forward(p: Params, num_seqs, q_pos0, nq, q, idx_q, idx_w, cache_cap, cache_len, proxy_k,
                 comp_logits, k_cache, v_cache, merged_f32, store, sel, sel_count, out, workspace,
                 stream=None):
    _ok(_lib.sgqa_forward(ctypes.byref(p.c()), num_seqs, q_pos0, nq, _ptr(q), _ptr(idx_q), _ptr(idx_w),
                          cache_cap, cache_len, _ptr(proxy_k), _ptr(comp_logits), _ptr(k_cache),
                          _ptr(v_cache), _ptr(merged_f32), _ptr(store), _ptr(sel), _ptr(sel_count),
                          _ptr(out), _ptr(workspace), workspace.numel() if workspace is not None else 0,
                          _stream(stream)))


def sgqa_sparse_attn_paged(p: Params, num_seqs, q_pos0, nq, q, k_pool, v_pool, page_table, cache_len, sel,
                           sel_count, out, gate=None, workspace=None, stream=None):
    """Attention over a paged cache: pools [num_pages, G, 16, D], page_table [S, max_pages] int32;
    a workspace only for calls of more than 32 queries per sequence."""
    num_pages = k_pool.shape[0]
    _ok(_lib.sgqa_sparse_attn_paged(ctypes.byref(p.c()), num_seqs, q_pos0, nq, _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                    num_pages, _ptr(page_table), page_table.shape[1], cache_len, _ptr(sel),
                                    _ptr(sel_count), _ptr(gate), _ptr(out), _ptr(workspace),
                                    workspace.numel() if workspace is not None else 0, _stream(stream)))


def sgqa_sparse_attn_noalloc(p: Params, num_seqs, q_pos0, nq, q, cache_cap, cache_len, k_cache, v_cache, sel,
                             sel_count, out, stream=None):
    """sgqa_sparse_attn for decode-sized calls (nq <= 32) using the library's
    static scratch instead of a workspace; for callers that cannot allocate."""
    _ok(_lib.sgqa_sparse_attn_noalloc(ctypes.byref(p.c()), num_seqs, q_pos0, nq, _ptr(q), cache_cap, cache_len,
                                      _ptr(k_cache), _ptr(v_cache), _ptr(sel), _ptr(sel_count), _ptr(out),
                                      _stream(stream)))


def sgqa_set_wait_limit_ns(ns: int):
    """Time limit of the kernels' pipeline waits on the current device (0: the default, 2 s)."""
    _ok(_lib.sgqa_set_wait_limit_ns(int(ns)))


def sgqa_check(stream=None):
    _ok(_lib.sgqa_check(_stream(stream)))
