"""Python front of the fp64 oracle -- TEST INFRASTRUCTURE ONLY.

Loads ``liboracle.so`` (built from ``tls_oracle.c`` with gcc; ``build()`` compiles
it on demand) and exposes numpy-level functions.  Only the tests, the smoke
check and the benchmark's CPU-baseline leg may import this module.  It imports
nothing from the CUDA package.

Each function restates one step of the AsyncTLS two-level sparse attention
(see the citations in ``tls_oracle.c``).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tls_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


class OraShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "batch", "n_q_heads", "n_kv_heads", "d_qk", "d_v", "v_is_k_prefix",
        "block_size", "n_label", "k_b", "k_t", "max_ctx", "dtype", "block_agg", "slab_bits")] + [
            ("softmax_scale", ctypes.c_double)]


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (plain C, gcc)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        S = ctypes.POINTER(OraShape)
        i = ctypes.c_int
        L.ora_abi_version.restype = i
        L.ora_build_meta.argtypes = [S, P, P, P]
        L.ora_block_scores.argtypes = [S, P, P, P, P]
        L.ora_topk.argtypes = [P, P, i, i, i, P, i]
        L.ora_topk.restype = i
        L.ora_select_blocks.argtypes = [S, P, P, i, P]
        L.ora_token_scores.argtypes = [S, P, P, P, P, P, P, P]
        L.ora_select_tokens.argtypes = [S, P, P, i, P]
        L.ora_attention.argtypes = [S, P, P, P, P, P, P]
        L.ora_decode_step.argtypes = [S, P, P, P, P, P, P, i, P, P, P, P]
        L.ora_quantize_labels.argtypes = [S, P, P, P, P, P]
        for f in ("ora_build_meta", "ora_block_scores", "ora_select_blocks", "ora_token_scores",
                  "ora_select_tokens", "ora_attention", "ora_decode_step", "ora_quantize_labels"):
            getattr(L, f).restype = None
        _lib = L
    return _lib


def shape_of(w, k_b: Optional[int] = None, k_t: Optional[int] = None, softmax_scale: Optional[float] = None):
    """OraShape from a workload description (attribute names as in workloads.Workload)."""
    s = OraShape()
    s.batch, s.n_q_heads, s.n_kv_heads = w.batch, w.n_q_heads, w.n_kv_heads
    s.d_qk, s.d_v, s.v_is_k_prefix = w.d_qk, w.d_v, int(w.v_is_k_prefix)
    s.block_size, s.n_label = w.block_size, w.n_label
    s.k_b = w.k_b if k_b is None else k_b
    s.k_t = w.k_t if k_t is None else k_t
    s.max_ctx, s.dtype = w.ctx, w.dtype
    s.block_agg = int(getattr(w, "block_agg", 0))
    s.slab_bits = int(getattr(w, "slab_bits", 0))
    s.softmax_scale = (1.0 / math.sqrt(w.d_qk)) if softmax_scale is None else softmax_scale
    return s


def _p(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _nbm(s) -> int:
    return -(-s.max_ctx // s.block_size)


def build_meta(s, K, seq_lens) -> np.ndarray:
    meta = np.empty((s.batch, s.n_kv_heads, _nbm(s), 2, s.d_qk), np.float64)
    lib().ora_build_meta(ctypes.byref(s), _p(K), _p(np.ascontiguousarray(seq_lens, np.int32)), _p(meta))
    return meta


def block_scores(s, q, meta, seq_lens) -> np.ndarray:
    out = np.empty((s.batch, s.n_kv_heads, _nbm(s)), np.float64)
    lib().ora_block_scores(ctypes.byref(s), _p(q), _p(np.ascontiguousarray(meta, np.float64)),
                           _p(np.ascontiguousarray(seq_lens, np.int32)), _p(out))
    return out


def topk(score, k: int, ids=None, decide_f32: bool = False, out_cap: Optional[int] = None):
    score = np.ascontiguousarray(score, np.float64)
    n = score.shape[0]
    ids_a = None if ids is None else np.ascontiguousarray(ids, np.int32)
    cap = k if out_cap is None else out_cap
    out = np.empty(max(cap, 1), np.int32)
    m = lib().ora_topk(_p(score), _p(ids_a), n, k, int(decide_f32), _p(out), cap)
    return out[:cap], m


def select_blocks(s, score, seq_lens, decide_f32: bool = False) -> np.ndarray:
    out = np.empty((s.batch, s.n_kv_heads, s.k_b), np.int32)
    lib().ora_select_blocks(ctypes.byref(s), _p(np.ascontiguousarray(score, np.float64)),
                            _p(np.ascontiguousarray(seq_lens, np.int32)), int(decide_f32), _p(out))
    return out


def token_scores(s, q, K, label_idx, block_idx, seq_lens):
    C = s.k_b * s.block_size
    sc = np.empty((s.batch, s.n_kv_heads, C), np.float64)
    tok = np.empty((s.batch, s.n_kv_heads, C), np.int32)
    lib().ora_token_scores(ctypes.byref(s), _p(q), _p(K), _p(np.ascontiguousarray(label_idx, np.int32)),
                           _p(np.ascontiguousarray(block_idx, np.int32)),
                           _p(np.ascontiguousarray(seq_lens, np.int32)), _p(sc), _p(tok))
    return sc, tok


def select_tokens(s, cand_score, cand_tok, decide_f32: bool = False) -> np.ndarray:
    out = np.empty((s.batch, s.n_kv_heads, s.k_t), np.int32)
    lib().ora_select_tokens(ctypes.byref(s), _p(np.ascontiguousarray(cand_score, np.float64)),
                            _p(np.ascontiguousarray(cand_tok, np.int32)), int(decide_f32), _p(out))
    return out


def attention(s, q, K, V, token_idx):
    out = np.empty((s.batch, s.n_q_heads, s.d_v), np.float64)
    lse = np.empty((s.batch, s.n_q_heads), np.float64)
    lib().ora_attention(ctypes.byref(s), _p(q), _p(K), _p(V), _p(np.ascontiguousarray(token_idx, np.int32)),
                        _p(out), _p(lse))
    return out, lse


def decode_step(s, q, K, V, meta, seq_lens, label_idx, decide_f32: bool = False, want_attention: bool = True):
    """Steps 2-6 chained.  Returns (block_idx, token_idx, out, lse)."""
    bidx = np.empty((s.batch, s.n_kv_heads, s.k_b), np.int32)
    tidx = np.empty((s.batch, s.n_kv_heads, s.k_t), np.int32)
    out = np.empty((s.batch, s.n_q_heads, s.d_v), np.float64) if want_attention else None
    lse = np.empty((s.batch, s.n_q_heads), np.float64) if want_attention else None
    lib().ora_decode_step(ctypes.byref(s), _p(q), _p(K), _p(V), _p(np.ascontiguousarray(meta, np.float64)),
                          _p(np.ascontiguousarray(seq_lens, np.int32)),
                          _p(np.ascontiguousarray(label_idx, np.int32)), int(decide_f32),
                          _p(bidx), _p(tidx), _p(out), _p(lse))
    return bidx, tidx, out, lse


def quantize_labels(s, K, seq_lens, label_idx):
    """The int8 label codes and their per-channel scales (the quantised slab
    reading); returns (codes [B][H_kv][max_ctx][r] int8, scales [B][H_kv][r] fp32)."""
    codes = np.empty((s.batch, s.n_kv_heads, s.max_ctx, s.n_label), np.int8)
    scales = np.empty((s.batch, s.n_kv_heads, s.n_label), np.float32)
    lib().ora_quantize_labels(ctypes.byref(s), _p(K), _p(np.ascontiguousarray(seq_lens, np.int32)),
                              _p(np.ascontiguousarray(label_idx, np.int32)), _p(codes), _p(scales))
    return codes, scales


def label_slab(s, K, label_idx) -> np.ndarray:
    """The label-channel slab K[..., L] (a plain gather of the stored values)."""
    return np.ascontiguousarray(K[..., np.asarray(label_idx, np.int64)])


def stream_decode(s, q_steps, K, V, meta, seq_lens, label_idx, decide_f32: bool = False):
    """Offloaded decode stream (gist.science (de) section 2.B; (es) section 2.B).

    Reading: at step t the block selection S_b(t) is computed from q_t (it is
    what the prefetch brings in for the next step), while token selection and
    attention at step t run inside S_b(t-1), the blocks already resident; step 0
    attends inside S_b(0).  Returns per-step lists of S_b(t), token_idx(t),
    out(t), lse(t) and the number of blocks new in S_b(t) relative to S_b(t-1).
    """
    T = q_steps.shape[0]
    res = {"block_idx": [], "token_idx": [], "out": [], "lse": [], "n_new": []}
    prev = None
    for t in range(T):
        q = np.ascontiguousarray(q_steps[t])
        sc = block_scores(s, q, meta, seq_lens)
        cur = select_blocks(s, sc, seq_lens, decide_f32)
        attend_in = cur if prev is None else prev
        cs, ct = token_scores(s, q, K, label_idx, attend_in, seq_lens)
        tidx = select_tokens(s, cs, ct, decide_f32)
        out, lse = attention(s, q, K, V, tidx)
        if prev is None:
            n_new = (cur >= 0).sum(axis=-1).astype(np.int32)
        else:
            n_new = np.zeros(cur.shape[:2], np.int32)
            for b in range(cur.shape[0]):
                for g in range(cur.shape[1]):
                    a = set(cur[b, g][cur[b, g] >= 0].tolist())
                    p = set(prev[b, g][prev[b, g] >= 0].tolist())
                    n_new[b, g] = len(a - p)
        res["block_idx"].append(cur)
        res["token_idx"].append(tidx)
        res["out"].append(out)
        res["lse"].append(lse)
        res["n_new"].append(n_new)
        prev = cur
    return res
