"""ctypes binding of libtls.so (include/tls.h): argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch
tensors (or raw integer pointers) and passes their device pointers, sizes and
the CUDA stream through unchanged.  No step of the decode path runs in Python;
a missing library raises ImportError at import time, and a failing call raises
TlsError with the library's message.  There is no fallback path.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtls.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python -m two_level_sparse_quest_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

TLS_OK, TLS_ERR_INVALID_ARG, TLS_ERR_UNSUPPORTED, TLS_ERR_WORKSPACE, TLS_ERR_CUDA, TLS_ERR_TIMEOUT = range(6)
TLS_F32, TLS_BF16 = 0, 1
STATUS_NAMES = {0: "TLS_OK", 1: "TLS_ERR_INVALID_ARG", 2: "TLS_ERR_UNSUPPORTED", 3: "TLS_ERR_WORKSPACE",
                4: "TLS_ERR_CUDA", 5: "TLS_ERR_TIMEOUT"}

EXPORTED = ("tls_version", "tls_last_error", "tls_workspace_size", "tls_build_block_meta", "tls_block_score_topk",
            "tls_token_score_topk", "tls_sparse_attn_decode", "tls_sparse_attn_decode_paged", "tls_offload_reset",
            "tls_prefetch_diff", "tls_wait_event", "tls_block_score_topk_noalloc", "tls_device_error", "tls_select_step",
            "tls_append_tokens", "tls_slab_bytes", "tls_noalloc_read_scores", "tls_decode_step", "tls_select_step_ws")


class TlsShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "n_q_heads", "n_kv_heads", "d_qk", "d_v", "v_is_k_prefix", "block_size", "n_label",
        "k_b", "k_t", "max_ctx", "kv_dtype", "out_dtype")] + [("softmax_scale", ctypes.c_float),
                                                               ("block_agg", ctypes.c_int32),
                                                               ("slab_bits", ctypes.c_int32)]

    def __repr__(self):
        return "TlsShape(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class TlsError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_P = ctypes.c_void_p
_S = ctypes.POINTER(TlsShape)
_i32 = ctypes.c_int32
_sz = ctypes.c_size_t
_sigs = {
    "tls_version": ([], ctypes.c_char_p),
    "tls_last_error": ([], ctypes.c_char_p),
    "tls_workspace_size": ([_S], _sz),
    "tls_build_block_meta": ([_S, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "tls_block_score_topk": ([_S, _P, _P, _P, _P, _P, _P, _sz, _P], ctypes.c_int),
    "tls_token_score_topk": ([_S, _P, _P, _P, _P, _P, _P, _P, _P, _sz, _P], ctypes.c_int),
    "tls_sparse_attn_decode": ([_S, _P, _P, _P, _P, _P, _P, _P, _sz, _P], ctypes.c_int),
    "tls_sparse_attn_decode_paged": ([_S, _P, _P, _P, _i32, _P, _P, _P, _P, _sz, _P], ctypes.c_int),
    "tls_offload_reset": ([_S, _i32, _P, _P, _P], ctypes.c_int),
    "tls_prefetch_diff": ([_S, _i32, _P, _P, _P, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "tls_wait_event": ([_P, _i32], ctypes.c_int),
    "tls_block_score_topk_noalloc": ([_S, _P, _P, _P, _P, _P], ctypes.c_int),
    "tls_device_error": ([ctypes.POINTER(_i32), _i32], ctypes.c_int),
    "tls_select_step": ([_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "tls_append_tokens": ([_S, _P, _P, _P, _i32, _P, _P, _P, _P], ctypes.c_int),
    "tls_slab_bytes": ([_S], _sz),
    "tls_noalloc_read_scores": ([_P, _sz, _P], ctypes.c_int),
    "tls_decode_step": ([_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _sz, _P], ctypes.c_int),
    "tls_select_step_ws": ([_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _sz, _P], ctypes.c_int),
}
for _name, (_args, _ret) in _sigs.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _ret


def make_shape(batch, n_q_heads, n_kv_heads, d_qk, d_v, block_size, n_label, k_b, k_t, max_ctx, kv_dtype,
               out_dtype=TLS_F32, v_is_k_prefix=False, softmax_scale: Optional[float] = None,
               block_agg: int = 0, slab_bits: int = 0) -> TlsShape:
    s = TlsShape()
    s.batch, s.n_q_heads, s.n_kv_heads = batch, n_q_heads, n_kv_heads
    s.d_qk, s.d_v, s.v_is_k_prefix = d_qk, d_v, int(bool(v_is_k_prefix))
    s.block_size, s.n_label, s.k_b, s.k_t, s.max_ctx = block_size, n_label, k_b, k_t, max_ctx
    s.kv_dtype, s.out_dtype = kv_dtype, out_dtype
    s.softmax_scale = (1.0 / math.sqrt(d_qk)) if softmax_scale is None else softmax_scale
    s.block_agg = int(block_agg)
    s.slab_bits = int(slab_bits)
    return s


def shape_from_workload(w, out_dtype=TLS_F32, **over) -> TlsShape:
    kw = dict(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, d_qk=w.d_qk, d_v=w.d_v,
              block_size=w.block_size, n_label=w.n_label, k_b=w.k_b, k_t=w.k_t, max_ctx=w.ctx, kv_dtype=w.dtype,
              out_dtype=out_dtype, v_is_k_prefix=w.v_is_k_prefix, block_agg=getattr(w, "block_agg", 0),
              slab_bits=getattr(w, "slab_bits", 0))
    kw.update(over)
    return make_shape(**kw)


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, torch.Tensor):
        if not x.is_contiguous():
            raise ValueError("tensor must be contiguous")
        return x.data_ptr()
    raise TypeError(f"expected a tensor, an int pointer or None, got {type(x)}")


def _dptr(x):
    """Pointer of an argument the kernels read or write on the device: a CUDA
    tensor (a host tensor is refused here, before it could reach a kernel) or
    a raw integer pointer, passed as is."""
    if isinstance(x, torch.Tensor) and x.device.type != "cuda":
        raise ValueError("expected a CUDA tensor (the kernels address device memory)")
    return _ptr(x)


def _hptr(x):
    """Pointer of host memory that a kernel reads directly: pinned (page-locked)."""
    if isinstance(x, torch.Tensor) and x.device.type != "cuda" and not x.is_pinned():
        raise ValueError("host_kv must be pinned host memory (torch.Tensor.pin_memory())")
    return _ptr(x)


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ws(ws):
    if ws is None:
        return None, 0
    if isinstance(ws, tuple):
        return ws
    return _dptr(ws), ws.numel() * ws.element_size()


def _check(st: int, name: str):
    if st != TLS_OK:
        raise TlsError(st, f"{name}: {tls_last_error()}")


def tls_version() -> str:
    return _lib.tls_version().decode()


def tls_last_error() -> str:
    return _lib.tls_last_error().decode()


def tls_workspace_size(shape: TlsShape) -> int:
    n = _lib.tls_workspace_size(ctypes.byref(shape))
    if n == 0:
        raise TlsError(TLS_ERR_UNSUPPORTED, f"tls_workspace_size: {tls_last_error()}")
    return n


def tls_slab_bytes(shape: TlsShape) -> int:
    n = _lib.tls_slab_bytes(ctypes.byref(shape))
    if n == 0:
        raise TlsError(TLS_ERR_UNSUPPORTED, f"tls_slab_bytes: {tls_last_error()}")
    return n


def tls_build_block_meta(shape, K, seq_lens, label_idx, meta_out, slab_out=None, stream=None):
    _check(_lib.tls_build_block_meta(ctypes.byref(shape), _dptr(K), _dptr(seq_lens), _dptr(label_idx), _dptr(meta_out),
                                     _dptr(slab_out), _stream(stream)), "tls_build_block_meta")


def tls_append_tokens(shape, K, old_lens, new_lens, max_append, label_idx, meta_out, slab_out=None, stream=None):
    _check(_lib.tls_append_tokens(ctypes.byref(shape), _dptr(K), _dptr(old_lens), _dptr(new_lens), int(max_append),
                                  _dptr(label_idx), _dptr(meta_out), _dptr(slab_out), _stream(stream)),
           "tls_append_tokens")


def tls_block_score_topk(shape, q, meta, seq_lens, block_idx_out, block_score_out=None, ws=None, stream=None):
    wp, wb = _ws(ws)
    _check(_lib.tls_block_score_topk(ctypes.byref(shape), _dptr(q), _dptr(meta), _dptr(seq_lens), _dptr(block_idx_out),
                                     _dptr(block_score_out), wp, wb, _stream(stream)), "tls_block_score_topk")


def tls_token_score_topk(shape, q, slab, label_idx, block_idx, seq_lens, token_idx_out, token_score_out=None,
                         ws=None, stream=None):
    wp, wb = _ws(ws)
    _check(_lib.tls_token_score_topk(ctypes.byref(shape), _dptr(q), _dptr(slab), _dptr(label_idx), _dptr(block_idx),
                                     _dptr(seq_lens), _dptr(token_idx_out), _dptr(token_score_out), wp, wb,
                                     _stream(stream)), "tls_token_score_topk")


def tls_select_step(shape, q, meta, slab, label_idx, seq_lens, block_idx_out, token_idx_out, block_score_out=None,
                    token_score_out=None, stream=None):
    _check(_lib.tls_select_step(ctypes.byref(shape), _dptr(q), _dptr(meta), _dptr(slab), _dptr(label_idx),
                                _dptr(seq_lens), _dptr(block_idx_out), _dptr(token_idx_out), _dptr(block_score_out),
                                _dptr(token_score_out), _stream(stream)), "tls_select_step")


def tls_select_step_ws(shape, q, meta, slab, label_idx, seq_lens, block_idx_out, token_idx_out, ws,
                       block_score_out=None, token_score_out=None, stream=None):
    """tls_select_step with tls_decode_step's workspace (the same launches as
    the selection part of tls_decode_step)."""
    wp, wn = _ws(ws)
    _check(_lib.tls_select_step_ws(ctypes.byref(shape), _dptr(q), _dptr(meta), _dptr(slab), _dptr(label_idx),
                                   _dptr(seq_lens), _dptr(block_idx_out), _dptr(token_idx_out),
                                   _dptr(block_score_out), _dptr(token_score_out), wp, wn, _stream(stream)),
           "tls_select_step_ws")


def tls_decode_step(shape, q, meta, slab, label_idx, seq_lens, K, V, block_idx_out, token_idx_out, out, lse_out=None,
                    block_score_out=None, token_score_out=None, ws=None, stream=None):
    """Stages 1-5 in one call (one launch for bf16 GQA shapes); ws must have
    been zero-filled before its first use by this call."""
    wp, wn = _ws(ws)
    _check(_lib.tls_decode_step(ctypes.byref(shape), _dptr(q), _dptr(meta), _dptr(slab), _dptr(label_idx),
                                _dptr(seq_lens), _dptr(K), _dptr(V), _dptr(block_idx_out), _dptr(token_idx_out),
                                _dptr(out), _dptr(lse_out), _dptr(block_score_out), _dptr(token_score_out), wp, wn,
                                _stream(stream)), "tls_decode_step")


def tls_sparse_attn_decode(shape, q, K, V, token_idx, out, lse_out=None, ws=None, stream=None):
    wp, wb = _ws(ws)
    _check(_lib.tls_sparse_attn_decode(ctypes.byref(shape), _dptr(q), _dptr(K), _dptr(V), _dptr(token_idx), _dptr(out),
                                       _dptr(lse_out), wp, wb, _stream(stream)), "tls_sparse_attn_decode")


def tls_sparse_attn_decode_paged(shape, q, cache, slot_of_block, n_slots, token_idx, out, lse_out=None, ws=None,
                                 stream=None):
    wp, wb = _ws(ws)
    _check(_lib.tls_sparse_attn_decode_paged(ctypes.byref(shape), _dptr(q), _dptr(cache), _dptr(slot_of_block),
                                             int(n_slots), _dptr(token_idx), _dptr(out), _dptr(lse_out), wp, wb,
                                             _stream(stream)), "tls_sparse_attn_decode_paged")


def tls_offload_reset(shape, n_slots, slot_of_block, block_of_slot, stream=None):
    _check(_lib.tls_offload_reset(ctypes.byref(shape), int(n_slots), _dptr(slot_of_block), _dptr(block_of_slot),
                                  _stream(stream)), "tls_offload_reset")


def tls_prefetch_diff(shape, n_slots, host_kv, cache, slot_of_block, block_of_slot, prev_block_idx, next_block_idx,
                      n_new_out, jobs_ws, stream=None):
    _check(_lib.tls_prefetch_diff(ctypes.byref(shape), int(n_slots), _hptr(host_kv), _dptr(cache), _dptr(slot_of_block),
                                  _dptr(block_of_slot), _dptr(prev_block_idx), _dptr(next_block_idx), _dptr(n_new_out),
                                  _dptr(jobs_ws), _stream(stream)), "tls_prefetch_diff")


def tls_block_score_topk_noalloc(shape, q, meta, seq_lens, block_idx_out, stream=None):
    """Block selection without a workspace, for callers that cannot allocate
    device memory: the scores live in a fixed array inside the library (see
    include/tls.h for the size limit and the sharing rules)."""
    _check(_lib.tls_block_score_topk_noalloc(ctypes.byref(shape), _dptr(q), _dptr(meta), _dptr(seq_lens),
                                             _dptr(block_idx_out), _stream(stream)), "tls_block_score_topk_noalloc")


def tls_noalloc_read_scores(dst, count: int, stream=None):
    """Copies the first `count` block scores that the last
    tls_block_score_topk_noalloc call left in the library's array into dst."""
    _check(_lib.tls_noalloc_read_scores(_dptr(dst), int(count), _stream(stream)), "tls_noalloc_read_scores")


def tls_wait_event(event, timeout_ms: int) -> int:
    """Returns the status (TLS_OK or TLS_ERR_TIMEOUT); raises on other errors."""
    handle = event if isinstance(event, int) else event.cuda_event
    st = _lib.tls_wait_event(handle, int(timeout_ms))
    if st not in (TLS_OK, TLS_ERR_TIMEOUT):
        _check(st, "tls_wait_event")
    return st


def tls_device_error(clear: bool = False) -> int:
    """Failure flags of the current device (1: an attention wait gave up,
    2: a selection exchange wait gave up); 0 means none since the last clear."""
    v = _i32(0)
    _check(_lib.tls_device_error(ctypes.byref(v), int(bool(clear))), "tls_device_error")
    return v.value
