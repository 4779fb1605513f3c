"""Seeded synthetic decode-step workloads (shared input generator).

This module is the only code that both the CUDA path and the fp64 oracle see.
It draws random numbers and encodes them (fp32 -> bf16 round-to-nearest-even);
it holds none of the two-level sparse attention arithmetic.

The shapes follow the workloads the AsyncTLS pages evaluate on: Qwen3-8B-shaped
GQA heads (32 query / 8 KV heads, head_dim 128) and a GLM-4.7-Flash-style
latent-attention layout (64 query heads sharing one 576-channel latent whose
first 512 channels serve as values), at 48k-96k contexts ("AsyncTLS" abstract,
mlsanity.com; gist.science explainers, section 4).  The pages measure on RULER /
LongBench with trained weights; these seeded Gaussian inputs with planted
outlier channels and needle keys stand in for those inputs and for nothing else.

Structure of every workload:
  * q ~ N(0, 1) per query head.
  * K ~ N(0, 1) with a fixed set of outlier channels scaled by ``outlier_scale``
    (a model property: the same channels for every sequence and KV head).
  * V ~ N(0, 1) (latent attention: V is the first d_v channels of K).
  * ``n_needles`` key rows per KV head replaced by 4 * qbar / |qbar|, where qbar
    is the sum of the (already rounded) query rows of the heads sharing that KV
    head, so that selection is non-trivial.  Needles are written after outlier
    scaling.
  * The label-channel set L (Double-Sparsity "label channels") is an input of the
    method; the generator returns the planted outlier channels plus a seeded
    random choice of the remaining channels, sorted ascending.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Optional

import numpy as np

F32 = 0
BF16 = 1


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    d_qk: int
    d_v: int
    v_is_k_prefix: bool
    ctx: int
    block_size: int
    k_b: int
    k_t: int
    n_label: int
    dtype: int
    n_outlier: int
    outlier_scale: float
    n_needles: int
    seed: int
    steps: int = 1          # decode steps (> 1 only for the AR(1) query stream)
    block_agg: int = 0      # block score over the group's heads: 0 sum (the method), 1 max (variant)
    slab_bits: int = 0      # label slab: 0 the K dtype, 8 int8 codes with per-channel scales (variant)
    ar_rho: float = 0.0     # q_t = rho q_{t-1} + sqrt(1 - rho^2) N(0, I)

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_blocks(self) -> int:
        return -(-self.ctx // self.block_size)

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == F32 else 2

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five decode workloads.  Names describe shape and context.
WORKLOADS = {
    "tiny_gqa4k_f32": Workload(
        "tiny_gqa4k_f32", batch=1, n_q_heads=4, n_kv_heads=1, d_qk=64, d_v=64,
        v_is_k_prefix=False, ctx=4096, block_size=32, k_b=16, k_t=256, n_label=16,
        dtype=F32, n_outlier=0, outlier_scale=1.0, n_needles=3, seed=1001),
    "gqa48k_bf16": Workload(
        "gqa48k_bf16", batch=1, n_q_heads=32, n_kv_heads=8, d_qk=128, d_v=128,
        v_is_k_prefix=False, ctx=49152, block_size=32, k_b=192, k_t=2048, n_label=16,
        dtype=BF16, n_outlier=8, outlier_scale=5.0, n_needles=16, seed=1002),
    "gqa96k_b8_bf16": Workload(
        "gqa96k_b8_bf16", batch=8, n_q_heads=32, n_kv_heads=8, d_qk=128, d_v=128,
        v_is_k_prefix=False, ctx=98304, block_size=32, k_b=256, k_t=4096, n_label=16,
        dtype=BF16, n_outlier=8, outlier_scale=5.0, n_needles=16, seed=1003),
    "mla64k_b4_bf16": Workload(
        "mla64k_b4_bf16", batch=4, n_q_heads=64, n_kv_heads=1, d_qk=576, d_v=512,
        v_is_k_prefix=True, ctx=65536, block_size=64, k_b=128, k_t=2048, n_label=32,
        dtype=BF16, n_outlier=16, outlier_scale=4.0, n_needles=32, seed=1004),
    "stream96k_bf16": Workload(
        "stream96k_bf16", batch=1, n_q_heads=32, n_kv_heads=8, d_qk=128, d_v=128,
        v_is_k_prefix=False, ctx=98304, block_size=32, k_b=192, k_t=2048, n_label=16,
        dtype=BF16, n_outlier=8, outlier_scale=5.0, n_needles=16, seed=1005,
        steps=128, ar_rho=0.9),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u >> np.uint32(16)) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r >>= np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact bf16 -> fp32 widening."""
    return (np.ascontiguousarray(b).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_f64(a: np.ndarray, dtype: int) -> np.ndarray:
    """Exact widening of stored input values (fp32 or bf16 bits) to fp64."""
    if dtype == BF16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def encode(x: np.ndarray, dtype: int) -> np.ndarray:
    """Store fp32 values in the workload dtype (bf16 as uint16 bits)."""
    if dtype == BF16:
        return f32_to_bf16_bits(x)
    return np.ascontiguousarray(x, dtype=np.float32)


def channel_sets(w: Workload):
    """Outlier channels and label channels (both sorted ascending, int32)."""
    rng = np.random.default_rng([w.seed, 1])
    outlier = np.sort(rng.choice(w.d_qk, size=w.n_outlier, replace=False)) if w.n_outlier else np.zeros(0, np.int64)
    rest = np.setdiff1d(np.arange(w.d_qk), outlier)
    rest = rng.permutation(rest)
    n_extra = max(0, w.n_label - len(outlier))
    label = np.sort(np.concatenate([outlier[: w.n_label], rest[:n_extra]]))
    return outlier.astype(np.int32), label.astype(np.int32)


@dataclass
class DecodeInputs:
    w: Workload
    q: np.ndarray            # [B][H_q][d_qk]   (uint16 bf16 bits or float32)
    K: np.ndarray            # [B][H_kv][ctx][d_qk]
    V: Optional[np.ndarray]  # [B][H_kv][ctx][d_v] or None when V = K[..., :d_v]
    seq_lens: np.ndarray     # int32 [B]
    label_idx: np.ndarray    # int32 [r]
    outlier_idx: np.ndarray  # int32
    needle_pos: np.ndarray   # int32 [B][H_kv][n_needles] (sorted)


def _queries(rng, w: Workload) -> np.ndarray:
    return rng.standard_normal((w.n_q_heads, w.d_qk), dtype=np.float32)


def make_decode_inputs(w: Workload, seq_lens=None, batches=None) -> DecodeInputs:
    """Generate one decode step's inputs.

    ``seq_lens``: optional per-sequence valid lengths (default: all ``w.ctx``).
    ``batches``: optional subset of batch rows to generate (others are zero);
    each row b is drawn from its own seed so any subset is reproducible.
    """
    B, Hq, Hkv, d, dv, n = w.batch, w.n_q_heads, w.n_kv_heads, w.d_qk, w.d_v, w.ctx
    G = w.group
    outlier, label = channel_sets(w)
    if seq_lens is None:
        seq_lens = np.full(B, n, np.int32)
    seq_lens = np.asarray(seq_lens, np.int32)
    assert seq_lens.shape == (B,) and (seq_lens >= 0).all() and (seq_lens <= n).all()
    edt = np.uint16 if w.dtype == BF16 else np.float32
    q = np.zeros((B, Hq, d), edt)
    K = np.zeros((B, Hkv, n, d), edt)
    V = None if w.v_is_k_prefix else np.zeros((B, Hkv, n, dv), edt)
    needles = np.full((B, Hkv, w.n_needles), -1, np.int32)
    rows = range(B) if batches is None else batches
    for b in rows:
        rng = np.random.default_rng([w.seed, 2, b])
        qb = encode(_queries(rng, w), w.dtype)
        q[b] = qb
        qf = to_f64(qb, w.dtype)
        for g in range(Hkv):
            kg = rng.standard_normal((n, d), dtype=np.float32)
            if len(outlier):
                kg[:, outlier] *= np.float32(w.outlier_scale)
            L = int(seq_lens[b])
            m = min(w.n_needles, L)
            if m > 0:
                pos = np.sort(rng.choice(L, size=m, replace=False))
                qbar = qf[g * G:(g + 1) * G].sum(axis=0)
                nrm = np.linalg.norm(qbar)
                if nrm > 0:
                    kg[pos] = (4.0 * qbar / nrm).astype(np.float32)
                needles[b, g, :m] = pos
            K[b, g] = encode(kg, w.dtype)
            del kg
            if V is not None:
                V[b, g] = encode(rng.standard_normal((n, dv), dtype=np.float32), w.dtype)
    return DecodeInputs(w, q, K, V, seq_lens, label, outlier, needles)


def make_query_stream(w: Workload, steps: Optional[int] = None) -> np.ndarray:
    """AR(1) query stream q_t = rho q_{t-1} + sqrt(1 - rho^2) N(0, I).

    Returns [steps][B][H_q][d_qk] in the workload dtype.  Step 0 equals the
    query of ``make_decode_inputs`` (same seed stream), so needles planted for
    step 0 stay aligned with the early queries.
    """
    T = w.steps if steps is None else steps
    B = w.batch
    rho = np.float32(w.ar_rho)
    sig = np.float32(np.sqrt(1.0 - w.ar_rho * w.ar_rho))
    out = np.zeros((T, B, w.n_q_heads, w.d_qk), np.uint16 if w.dtype == BF16 else np.float32)
    for b in range(B):
        q = _queries(np.random.default_rng([w.seed, 2, b]), w)
        rng = np.random.default_rng([w.seed, 3, b])
        for t in range(T):
            if t > 0:
                q = rho * q + sig * rng.standard_normal(q.shape, dtype=np.float32)
            out[t, b] = encode(q, w.dtype)
    return out


def paged_host_kv(inp: DecodeInputs) -> np.ndarray:
    """Host KV in block-major layout [B][H_kv][N_b][2][bs][d] (K block, then V block).

    Used by the offloaded stream: one block is one contiguous host range.  The
    tail of a partial last block is zero.
    """
    w = inp.w
    assert not w.v_is_k_prefix and w.d_qk == w.d_v
    B, Hkv, n, d, bs = w.batch, w.n_kv_heads, w.ctx, w.d_qk, w.block_size
    nb = w.n_blocks
    out = np.zeros((B, Hkv, nb, 2, bs, d), inp.K.dtype)
    pad = nb * bs - n
    for b in range(B):
        for g in range(Hkv):
            k = inp.K[b, g]
            v = inp.V[b, g]
            if pad:
                k = np.concatenate([k, np.zeros((pad, d), k.dtype)])
                v = np.concatenate([v, np.zeros((pad, d), v.dtype)])
            out[b, g, :, 0] = k.reshape(nb, bs, d)
            out[b, g, :, 1] = v.reshape(nb, bs, d)
    return out
