"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each pin checks the oracle against something the mathematics or the pages fix:
brute force on tiny inputs, closed forms, invariants (the block bound is an
upper bound and is attained at a corner of the box), special cases that reduce
to a library routine (full selection == torch scaled-dot-product attention in
fp64), and hand-worked examples stored under tests/golden/.
A final group plants mistakes in copies of the oracle and checks that the pins
catch them.
"""
import ctypes
import itertools
import json
import math
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from oracle import oracle as O
from two_level_sparse_quest_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


class Sh:
    """Minimal workload-like description for the oracle."""

    def __init__(self, **kw):
        self.__dict__.update(dict(batch=1, n_q_heads=1, n_kv_heads=1, d_qk=8, d_v=8, v_is_k_prefix=False,
                                  block_size=4, n_label=4, k_b=2, k_t=4, ctx=16, dtype=W.F32))
        self.__dict__.update(kw)


def rand_inputs(sh, seed, dtype=W.F32, seq_lens=None):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((sh.batch, sh.n_q_heads, sh.d_qk)).astype(np.float32)
    K = rng.standard_normal((sh.batch, sh.n_kv_heads, sh.ctx, sh.d_qk)).astype(np.float32)
    V = rng.standard_normal((sh.batch, sh.n_kv_heads, sh.ctx, sh.d_v)).astype(np.float32)
    if dtype == W.BF16:
        q, K, V = W.f32_to_bf16_bits(q), W.f32_to_bf16_bits(K), W.f32_to_bf16_bits(V)
    sl = np.full(sh.batch, sh.ctx, np.int32) if seq_lens is None else np.asarray(seq_lens, np.int32)
    return q, K, V, sl


def f64(a, dtype):
    return W.to_f64(a, dtype)


# --------------------------------------------------------------------------- meta
@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
def test_meta_equals_bruteforce_minmax(dtype):
    sh = Sh(batch=3, n_kv_heads=2, ctx=37, block_size=8, d_qk=5, dtype=dtype)
    q, K, V, sl = rand_inputs(sh, 1, dtype, seq_lens=[37, 20, 0])
    s = O.shape_of(sh)
    meta = O.build_meta(s, K, sl)
    Kf = f64(K, dtype)
    nbm = -(-sh.ctx // sh.block_size)
    for b in range(sh.batch):
        for g in range(sh.n_kv_heads):
            for j in range(nbm):
                t0, t1 = j * sh.block_size, min((j + 1) * sh.block_size, int(sl[b]))
                if t0 >= t1:
                    assert np.isnan(meta[b, g, j]).all()
                    continue
                blk = Kf[b, g, t0:t1]
                np.testing.assert_array_equal(meta[b, g, j, 0], blk.max(axis=0))
                np.testing.assert_array_equal(meta[b, g, j, 1], blk.min(axis=0))


# --------------------------------------------------------------------------- block bound
def per_head_bounds(sh, q, meta, sl):
    """Per-head bounds obtained by running the oracle on one head at a time."""
    out = []
    for h in range(sh.n_q_heads):
        g = h // (sh.n_q_heads // sh.n_kv_heads)
        one = Sh(**{**sh.__dict__, "n_q_heads": 1, "n_kv_heads": 1})
        s1 = O.shape_of(one)
        qh = np.ascontiguousarray(q[:, h:h + 1])
        mh = np.ascontiguousarray(meta[:, g:g + 1])
        out.append(O.block_scores(s1, qh, mh, sl)[:, 0])
    return np.stack(out, axis=1)  # [B][H_q][N_b]


@pytest.mark.parametrize("seed,heads", [(0, (4, 2)), (1, (4, 2)), (2, (4, 2)), (3, (32, 1)), (4, (1, 1))])
def test_block_bound_dominates_every_key(seed, heads):
    # GQA, MQA (32 query heads on one KV head) and MHA (one head per KV head)
    sh = Sh(batch=2, n_q_heads=heads[0], n_kv_heads=heads[1], ctx=40, block_size=8, d_qk=6)
    q, K, V, sl = rand_inputs(sh, seed, seq_lens=[40, 29])
    s = O.shape_of(sh)
    meta = O.build_meta(s, K, sl)
    score = O.block_scores(s, q, meta, sl)
    u = per_head_bounds(sh, q, meta, sl)
    Kf, qf = f64(K, W.F32), f64(q, W.F32)
    G = sh.n_q_heads // sh.n_kv_heads
    for b in range(sh.batch):
        nb = -(-int(sl[b]) // sh.block_size)
        assert np.isneginf(score[b, :, nb:]).all()
        for g in range(sh.n_kv_heads):
            for j in range(nb):
                toks = Kf[b, g, j * sh.block_size:min((j + 1) * sh.block_size, int(sl[b]))]
                dots = qf[b, g * G:(g + 1) * G] @ toks.T  # [G][tokens]
                for hh in range(G):
                    assert u[b, g * G + hh, j] >= dots[hh].max() - 1e-12
                # group score: sum of the per-head bounds, and above the best group dot
                assert score[b, g, j] == pytest.approx(u[b, g * G:(g + 1) * G, j].sum(), rel=1e-13, abs=1e-13)
                assert score[b, g, j] >= dots.sum(axis=0).max() - 1e-12


@pytest.mark.parametrize("seed", [0, 1])
def test_max_over_heads_aggregation_is_the_largest_single_head_bound(seed):
    """The aggregation variant: a group's block score is the largest of its
    heads' bounds, each obtained by running the oracle on that head alone; with
    one head per group both aggregations coincide."""
    sh = Sh(batch=2, n_q_heads=8, n_kv_heads=2, ctx=48, block_size=8, d_qk=6)
    q, K, V, sl = rand_inputs(sh, seed, seq_lens=[48, 21])
    meta = O.build_meta(O.shape_of(sh), K, sl)
    shm = Sh(**{**sh.__dict__, "block_agg": 1})
    smax = O.block_scores(O.shape_of(shm), q, meta, sl)
    ssum = O.block_scores(O.shape_of(sh), q, meta, sl)
    u = per_head_bounds(sh, q, meta, sl)  # [B][H_q][N_b]
    G = sh.n_q_heads // sh.n_kv_heads
    want = u.reshape(sh.batch, sh.n_kv_heads, G, -1).max(axis=2)
    np.testing.assert_array_equal(smax, want)
    assert not np.array_equal(np.nan_to_num(smax, neginf=0), np.nan_to_num(ssum, neginf=0))
    one = Sh(**{**sh.__dict__, "n_q_heads": 2, "n_kv_heads": 2})
    one_max = Sh(**{**one.__dict__, "block_agg": 1})
    q1 = np.ascontiguousarray(q[:, :2])
    np.testing.assert_array_equal(O.block_scores(O.shape_of(one), q1, meta, sl),
                                  O.block_scores(O.shape_of(one_max), q1, meta, sl))


def test_block_bound_is_attained_at_box_corner():
    # max of a linear function over a box is attained at the corner that follows sign(q)
    sh = Sh(n_q_heads=1, n_kv_heads=1, ctx=64, block_size=16, d_qk=9)
    for seed in range(5):
        q, K, V, sl = rand_inputs(sh, 10 + seed)
        s = O.shape_of(sh)
        meta = O.build_meta(s, K, sl)
        score = O.block_scores(s, q, meta, sl)
        qf = f64(q, W.F32)[0, 0]
        for j in range(4):
            corner = np.where(qf >= 0, meta[0, 0, j, 0], meta[0, 0, j, 1])
            assert score[0, 0, j] == pytest.approx(float(qf @ corner), rel=1e-13, abs=1e-13)
            # the corner lies inside the box and no other corner is higher
            for signs in itertools.islice(itertools.product([0, 1], repeat=sh.d_qk), 64):
                other = np.where(np.array(signs) == 1, meta[0, 0, j, 0], meta[0, 0, j, 1])
                assert float(qf @ other) <= score[0, 0, j] + 1e-12


def test_block_bound_with_block_size_one_is_exact_dot():
    sh = Sh(n_q_heads=3, n_kv_heads=1, ctx=11, block_size=1, d_qk=7)
    q, K, V, sl = rand_inputs(sh, 3)
    s = O.shape_of(sh)
    score = O.block_scores(s, q, O.build_meta(s, K, sl), sl)
    exact = (f64(q, W.F32)[0] @ f64(K, W.F32)[0, 0].T).sum(axis=0)
    np.testing.assert_allclose(score[0, 0], exact, rtol=1e-13, atol=1e-13)


def test_block_bound_adversarial_blocks():
    # constant channels, all-negative keys, zero query, one-token block
    sh = Sh(n_q_heads=2, n_kv_heads=1, ctx=9, block_size=4, d_qk=3)
    K = np.array([[[[2, -1, 0], [2, -3, 0], [2, -2, 0], [2, -1, 0],
                    [-5, -5, -5], [-6, -4, -5], [-5, -5, -7], [-9, -5, -5],
                    [1, 1, 1]]]], np.float32)
    q = np.array([[[1, -2, 3], [0, 0, 0]]], np.float32)
    sl = np.array([9], np.int32)
    s = O.shape_of(sh)
    score = O.block_scores(s, q, O.build_meta(s, K, sl), sl)
    # block 0: head0 = 1*2 + max(-2*-1, -2*-3)=6 + 0 = 8; head1 = 0
    # block 1: head0 = max(-5,-9) + max(8,10) + max(-15,-21) = -5 + 10 - 15 = -10
    # block 2: one token [1,1,1] -> head0 = 1 - 2 + 3 = 2
    np.testing.assert_array_equal(score[0, 0], [8.0, -10.0, 2.0])


# --------------------------------------------------------------------------- top-k
def brute_topk(scores, ids, k):
    n = len(scores)
    m = min(k, n)
    keyed = [(scores[i], -ids[i]) for i in range(n)]
    winners = []
    for sub in itertools.combinations(range(n), m):
        inside = set(sub)
        if all(keyed[a] > keyed[b] for a in inside for b in range(n) if b not in inside):
            winners.append(sorted(ids[a] for a in sub))
    assert len(winners) == 1  # unique maximiser
    return winners[0]


@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_bruteforce_with_ties(seed):
    rng = np.random.default_rng(seed)
    for n in range(0, 11):
        scores = rng.integers(-3, 4, size=n).astype(np.float64)  # many exact ties
        ids = rng.permutation(100)[:n].astype(np.int32)
        for k in range(0, n + 2):
            got, m = O.topk(scores, k, ids=ids, out_cap=k + 1)
            assert m == min(k, n)
            want = brute_topk(list(scores), list(ids), k) if n else []
            assert list(got[:m]) == want
            assert (got[m:] == -1).all()


def test_topk_decide_in_f32_rounds_before_ranking():
    # 1 + 2^-30 and 1 differ in fp64 but are equal in fp32 -> the lower id wins
    s = np.array([1.0, 1.0 + 2.0 ** -30], np.float64)
    got64, _ = O.topk(s, 1)
    got32, _ = O.topk(s, 1, decide_f32=True)
    assert list(got64) == [1] and list(got32) == [0]


# --------------------------------------------------------------------------- token scores
def test_token_scores_with_all_channels_equal_group_dot():
    sh = Sh(batch=2, n_q_heads=4, n_kv_heads=2, ctx=24, block_size=4, d_qk=6, n_label=6, k_b=3)
    q, K, V, sl = rand_inputs(sh, 5, seq_lens=[24, 14])
    s = O.shape_of(sh)
    bidx = np.array([[[5, 0, 2], [1, -1, -1]], [[3, 2, 1], [0, 1, 3]]], np.int32)
    sc, tok = O.token_scores(s, q, K, np.arange(6, dtype=np.int32), bidx, sl)
    qf, Kf = f64(q, W.F32), f64(K, W.F32)
    G = 2
    for b in range(2):
        for g in range(2):
            for j in range(3 * 4):
                blk = bidx[b, g, j // 4]
                t = blk * 4 + j % 4
                if blk < 0 or t >= sl[b]:
                    assert tok[b, g, j] == -1 and np.isneginf(sc[b, g, j])
                else:
                    assert tok[b, g, j] == t
                    want = float((qf[b, g * G:(g + 1) * G] @ Kf[b, g, t]).sum())
                    assert sc[b, g, j] == pytest.approx(want, rel=1e-13, abs=1e-13)


def test_token_scores_single_label_channel_is_product():
    sh = Sh(n_q_heads=2, n_kv_heads=1, ctx=8, block_size=4, d_qk=5, n_label=1, k_b=2)
    q, K, V, sl = rand_inputs(sh, 6)
    s = O.shape_of(sh)
    sc, tok = O.token_scores(s, q, K, np.array([3], np.int32), np.array([[[0, 1]]], np.int32), sl)
    qf, Kf = f64(q, W.F32), f64(K, W.F32)
    np.testing.assert_allclose(sc[0, 0], (qf[0, 0, 3] + qf[0, 1, 3]) * Kf[0, 0, :, 3], rtol=1e-15)


# --------------------------------------------------------------------------- attention
def sdpa_fp64(q, K, V, scale):
    """torch scaled_dot_product_attention in fp64 on CPU: q [H][d], K [n][d], V [n][dv]."""
    qt = torch.from_numpy(q)[None, :, None, :]
    kt = torch.from_numpy(K)[None, None].expand(1, q.shape[0], -1, -1)
    vt = torch.from_numpy(V)[None, None].expand(1, q.shape[0], -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    return o[0, :, 0].numpy()


@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
def test_full_selection_equals_full_attention(dtype):
    sh = Sh(batch=2, n_q_heads=6, n_kv_heads=2, ctx=48, block_size=8, d_qk=16, d_v=12, n_label=4,
            k_b=6, k_t=48, dtype=dtype)
    q, K, V, sl = rand_inputs(sh, 7, dtype, seq_lens=[48, 45])
    s = O.shape_of(sh)
    meta = O.build_meta(s, K, sl)
    bidx, tidx, out, lse = O.decode_step(s, q, K, V, meta, sl, np.arange(4, dtype=np.int32))
    qf, Kf, Vf = f64(q, dtype), f64(K, dtype), f64(V, dtype)
    G = 3
    for b in range(2):
        L = int(sl[b])
        for g in range(2):
            assert list(bidx[b, g]) == list(range(-(-L // 8)))
            assert list(tidx[b, g][:L]) == list(range(L)) and (tidx[b, g][L:] == -1).all()
            qg = qf[b, g * G:(g + 1) * G]
            ref = sdpa_fp64(qg, Kf[b, g, :L], Vf[b, g, :L], s.softmax_scale)
            np.testing.assert_allclose(out[b, g * G:(g + 1) * G], ref, rtol=1e-12, atol=1e-12)
            ref_lse = logsumexp(s.softmax_scale * qg @ Kf[b, g, :L].T, axis=1)
            np.testing.assert_allclose(lse[b, g * G:(g + 1) * G], ref_lse, rtol=1e-13, atol=1e-13)


def test_full_selection_latent_values_prefix():
    sh = Sh(n_q_heads=8, n_kv_heads=1, ctx=32, block_size=8, d_qk=20, d_v=16, v_is_k_prefix=True,
            n_label=4, k_b=4, k_t=32)
    q, K, V, sl = rand_inputs(sh, 8)
    s = O.shape_of(sh)
    meta = O.build_meta(s, K, sl)
    _, _, out, _ = O.decode_step(s, q, K, None, meta, sl, np.arange(4, dtype=np.int32))
    Kf = f64(K, W.F32)[0, 0]
    ref = sdpa_fp64(f64(q, W.F32)[0], Kf, np.ascontiguousarray(Kf[:, :16]), s.softmax_scale)
    np.testing.assert_allclose(out[0], ref, rtol=1e-12, atol=1e-12)


def test_two_token_closed_form_and_weights_sum_to_one():
    sh = Sh(n_q_heads=1, n_kv_heads=1, ctx=2, block_size=1, d_qk=3, d_v=2, k_b=2, k_t=2)
    q = np.array([[[0.5, -1.0, 2.0]]], np.float32)
    K = np.array([[[[1.0, 0.0, 0.25], [0.0, 2.0, -1.0]]]], np.float32)
    V = np.array([[[[3.0, -1.0], [1.0, 5.0]]]], np.float32)
    s = O.shape_of(sh, softmax_scale=0.75)
    out, lse = O.attention(s, q, K, V, np.array([[[0, 1]]], np.int32))
    a1, a2 = 0.75 * (0.5 + 0.5), 0.75 * (-2.0 - 2.0)
    w1 = 1.0 / (1.0 + math.exp(a2 - a1))
    np.testing.assert_allclose(out[0, 0], [w1 * 3 + (1 - w1) * 1, w1 * -1 + (1 - w1) * 5], rtol=1e-14)
    assert lse[0, 0] == pytest.approx(math.log(math.exp(a1) + math.exp(a2)), rel=1e-14)
    # scaling V scales the output; a convex combination never leaves [min V, max V]
    out2, _ = O.attention(s, q, K, 2 * V, np.array([[[0, 1]]], np.int32))
    np.testing.assert_allclose(out2, 2 * out, rtol=1e-15)


def test_attention_is_invariant_to_selection_order_and_padding():
    sh = Sh(n_q_heads=2, n_kv_heads=1, ctx=16, d_qk=4, d_v=4, k_t=6)
    q, K, V, sl = rand_inputs(sh, 9)
    s = O.shape_of(sh)
    a, la = O.attention(s, q, K, V, np.array([[[1, 4, 7, 9, -1, -1]]], np.int32))
    b, lb = O.attention(s, q, K, V, np.array([[[9, -1, 7, 1, -1, 4]]], np.int32))
    np.testing.assert_allclose(a, b, rtol=1e-14)
    np.testing.assert_allclose(la, lb, rtol=1e-14)


def test_attention_shift_invariance_with_large_logits():
    # Adding one vector v to every key moves every logit of head h by
    # tau * q_h.v: the output stays the same and lse moves by exactly that
    # amount, even when the shifted logits (~2048) would overflow exp in fp64
    # without the running-max subtraction.  Grid values keep every sum exact.
    sh = Sh(n_q_heads=2, n_kv_heads=1, ctx=16, d_qk=4, d_v=4, k_t=6)
    rng = np.random.default_rng(5)
    q = (rng.integers(-8, 9, (1, 2, 4)) / 8).astype(np.float32)
    q[0, :, 0] = [1.0, 0.5]
    K = (rng.integers(-16, 17, (1, 1, 16, 4)) / 16).astype(np.float32)
    V = rng.standard_normal((1, 1, 16, 4)).astype(np.float32)
    shift = np.array([2048.0, 0.0, 0.0, 0.0], np.float32)
    s = O.shape_of(sh, softmax_scale=1.0)
    idx = np.array([[[0, 3, 5, 8, 11, 15]]], np.int32)
    a, la = O.attention(s, q, K, V, idx)
    b, lb = O.attention(s, q, np.ascontiguousarray(K + shift), V, idx)
    assert np.isfinite(b).all() and np.isfinite(lb).all()
    np.testing.assert_allclose(b, a, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose((lb - la)[0], q[0, :, 0].astype(np.float64) * 2048.0, rtol=1e-12)


def test_empty_selection_gives_zero_output_and_neg_inf_lse():
    sh = Sh(n_q_heads=2, n_kv_heads=1, ctx=8, d_qk=4, d_v=4, k_t=3)
    q, K, V, sl = rand_inputs(sh, 11)
    s = O.shape_of(sh)
    out, lse = O.attention(s, q, K, V, np.full((1, 1, 3), -1, np.int32))
    assert (out == 0).all() and np.isneginf(lse).all()


def test_empty_sequence_selects_nothing():
    sh = Sh(batch=2, n_q_heads=2, n_kv_heads=1, ctx=16, d_qk=4, d_v=4, k_b=2, k_t=3)
    q, K, V, _ = rand_inputs(sh, 12)
    sl = np.array([0, 5], np.int32)
    s = O.shape_of(sh)
    meta = O.build_meta(s, K, sl)
    bidx, tidx, out, lse = O.decode_step(s, q, K, V, meta, sl, np.arange(4, dtype=np.int32))
    assert (bidx[0] == -1).all() and (tidx[0] == -1).all() and (out[0] == 0).all() and np.isneginf(lse[0]).all()
    assert list(bidx[1, 0]) == [0, 1] and (tidx[1, 0] >= 0).sum() == 3


# --------------------------------------------------------------------------- golden
def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _golden_shape(d):
    s = O.OraShape()
    for k, v in d["shape"].items():
        setattr(s, k, v)
    return s


def test_golden_hand_example_gqa2():
    d = _load("hand_example_gqa2.json")
    s = _golden_shape(d)
    q = np.array(d["q"], np.float32)[None]
    K = np.array(d["K"], np.float32)[None, None]
    V = np.array(d["V"], np.float32)[None, None]
    L = np.array(d["label_idx"], np.int32)
    sl = np.array([4], np.int32)
    e = d["expected"]
    meta = O.build_meta(s, K, sl)
    np.testing.assert_array_equal(meta[0, 0, :, 0], e["meta_max"])
    np.testing.assert_array_equal(meta[0, 0, :, 1], e["meta_min"])
    sc = O.block_scores(s, q, meta, sl)
    np.testing.assert_array_equal(sc[0, 0], e["block_scores"])
    bidx = O.select_blocks(s, sc, sl)
    assert list(bidx[0, 0]) == e["block_idx"]
    cs, ct = O.token_scores(s, q, K, L, bidx, sl)
    assert list(ct[0, 0]) == e["cand_tokens"]
    np.testing.assert_array_equal(cs[0, 0], e["cand_scores"])
    tidx = O.select_tokens(s, cs, ct)
    assert list(tidx[0, 0]) == e["token_idx"]
    out, lse = O.attention(s, q, K, V, tidx)
    sig = lambda x: 1.0 / (1.0 + math.exp(-x))
    (a0, a1), (c0, c1) = e["attention_logits"]
    v2, v3 = np.array(d["V"][2], float), np.array(d["V"][3], float)
    np.testing.assert_allclose(out[0, 0], sig(a0 - a1) * v2 + sig(a1 - a0) * v3, rtol=1e-14)
    np.testing.assert_allclose(out[0, 1], sig(c0 - c1) * v2 + sig(c1 - c0) * v3, rtol=1e-14)
    assert lse[0, 0] == pytest.approx(math.log(math.exp(a0) + math.exp(a1)), rel=1e-14)
    assert lse[0, 1] == pytest.approx(math.log(math.exp(c0) + math.exp(c1)), rel=1e-14)


def test_golden_tie_breaks_and_latent_values():
    d = _load("hand_example_tie_mla.json")
    s = _golden_shape(d)
    q = np.array(d["q"], np.float32)[None]
    K = np.array(d["K"], np.float32)[None, None]
    sl = np.array([6], np.int32)
    e = d["expected"]
    meta = O.build_meta(s, K, sl)
    sc = O.block_scores(s, q, meta, sl)
    np.testing.assert_array_equal(sc[0, 0], e["block_scores"])
    bidx, tidx, out, lse = O.decode_step(s, q, K, None, meta, sl, np.array(d["label_idx"], np.int32))
    assert list(bidx[0, 0]) == e["block_idx"] and list(tidx[0, 0]) == e["token_idx"]
    np.testing.assert_allclose(out[0], e["out"], rtol=1e-15)
    np.testing.assert_allclose(lse[0], e["lse"], rtol=1e-15)


# --------------------------------------------------------------------------- stream
def test_stream_constant_query_has_no_diff_after_first_step():
    w = W.WORKLOADS["tiny_gqa4k_f32"].with_(ctx=512, k_b=4, k_t=32)
    inp = W.make_decode_inputs(w)
    s = O.shape_of(w)
    meta = O.build_meta(s, inp.K, inp.seq_lens)
    qs = np.stack([inp.q] * 4)
    res = O.stream_decode(s, qs, inp.K, inp.V, meta, inp.seq_lens, inp.label_idx)
    assert res["n_new"][0].tolist() == [[4]]
    assert all(n.sum() == 0 for n in res["n_new"][1:])
    _, _, out, _ = O.decode_step(s, inp.q, inp.K, inp.V, meta, inp.seq_lens, inp.label_idx)
    for t in range(4):
        np.testing.assert_array_equal(res["out"][t], out)


def test_golden_stream_attends_inside_the_previous_selection():
    """Hand-worked three-step stream whose block selection changes every step:
    step t must attend inside S_b(t-1) (step 0 inside S_b(0)), so the outputs of
    steps 1 and 2 differ from attending inside the current or the first selection."""
    d = _load("stream_lag_three_steps.json")
    s = _golden_shape(d)
    qs = np.array(d["q_steps"], np.float32)[:, None, None, :]  # [T][B=1][H_q=1][d]
    K = np.array(d["K"], np.float32)[None, None]
    V = np.array(d["V"], np.float32)[None, None]
    sl = np.array([4], np.int32)
    L = np.array(d["label_idx"], np.int32)
    meta = O.build_meta(s, K, sl)
    res = O.stream_decode(s, qs, K, V, meta, sl, L)
    e = d["expected"]
    sig = lambda x: 1.0 / (1.0 + math.exp(-x))
    want_out = [[sig(1.0), sig(-1.0)], e["out"][1], e["out"][2]]
    want_lse = [math.log(math.exp(2.0) + math.exp(1.0)), math.log(2.0), math.log(2.0)]
    for t in range(3):
        assert res["block_idx"][t][0, 0].tolist() == e["block_idx"][t], f"S_b({t})"
        assert int(res["n_new"][t][0, 0]) == e["n_new"][t], f"new blocks at step {t}"
        assert res["token_idx"][t][0, 0].tolist() == e["token_idx"][t], f"tokens at step {t}"
        np.testing.assert_allclose(res["out"][t][0, 0], want_out[t], rtol=1e-14, atol=1e-15, err_msg=f"step {t}")
        assert res["lse"][t][0, 0] == pytest.approx(want_lse[t], rel=1e-14)


def test_needles_in_kept_blocks_win_token_selection():
    # workload diagnostic, not a parity claim: a planted needle key 4*qbar/|qbar| that sits
    # in a kept block scores far above random keys on the label channels and is kept
    w = W.WORKLOADS["tiny_gqa4k_f32"].with_(k_b=64)
    inp = W.make_decode_inputs(w)
    s = O.shape_of(w)
    meta = O.build_meta(s, inp.K, inp.seq_lens)
    bidx, tidx, _, _ = O.decode_step(s, inp.q, inp.K, inp.V, meta, inp.seq_lens, inp.label_idx, want_attention=False)
    kept_blocks = set(bidx[0, 0].tolist())
    kept_needles = [p for p in inp.needle_pos[0, 0].tolist() if p // w.block_size in kept_blocks]
    assert kept_needles, "no needle block kept; the diagnostic needs one"
    assert set(kept_needles) <= set(tidx[0, 0].tolist())


# --------------------------------------------------------------------------- planted mistakes
MUTANTS = {
    "bound_uses_min": ("u += (a > c) ? a : c;", "u += (a < c) ? a : c;"),
    "bound_drops_min_row": ("double a = qi * mx[i], c = qi * mn[i];", "double a = qi * mx[i], c = qi * mx[i];"),
    "token_score_wrong_channel": ("ora_in(K, s->dtype, (bg * s->max_ctx + t) * d + ch);",
                                  "ora_in(K, s->dtype, (bg * s->max_ctx + t) * d + c);"),
    "topk_ties_to_higher": ("return (a->id < b->id) ? -1 : (a->id > b->id);",
                            "return (a->id > b->id) ? -1 : (a->id < b->id);"),
    "softmax_drops_scale": ("a[j] = s->softmax_scale * acc;", "a[j] = acc;"),
    "meta_min_is_max": ("if (v < lo) lo = v;", "if (v > lo) lo = v;"),
}


def _mutant_lib(tmpdir, name):
    src = open(os.path.join(os.path.dirname(O.__file__), "tls_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    path = os.path.join(tmpdir, f"m_{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    so = path[:-2] + ".so"
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-shared", "-fPIC", path, "-o", so, "-lm"])
    return so


# Mistakes planted in the Python front (oracle.py) rather than the C file.
PY_MUTANTS = {
    "stream_attends_in_current": ("attend_in = cur if prev is None else prev", "attend_in = cur"),
    "stream_attends_in_first": ("attend_in = cur if prev is None else prev",
                                "attend_in = cur if prev is None else first"),
}

PIN_FOR_MUTANT = {
    "stream_attends_in_current": lambda: test_golden_stream_attends_inside_the_previous_selection(),
    "stream_attends_in_first": lambda: test_golden_stream_attends_inside_the_previous_selection(),
    "bound_uses_min": lambda: test_block_bound_dominates_every_key(0, (4, 2)),
    "bound_drops_min_row": lambda: test_block_bound_is_attained_at_box_corner(),
    "token_score_wrong_channel": lambda: test_token_scores_single_label_channel_is_product(),
    "topk_ties_to_higher": lambda: test_topk_matches_bruteforce_with_ties(0),
    "softmax_drops_scale": lambda: test_full_selection_equals_full_attention(W.F32),
    "meta_min_is_max": lambda: test_meta_equals_bruteforce_minmax(W.F32),
}


def _py_mutant_module(name):
    """A copy of oracle.py with one planted mistake, loaded as its own module
    (it loads the same, unmodified liboracle.so)."""
    import types

    src = open(O.__file__).read()
    old, new = PY_MUTANTS[name]
    assert src.count(old) == 1, name
    if name == "stream_attends_in_first":  # also remember the first selection
        src = src.replace("    prev = None\n", "    prev = None\n    first = None\n", 1)
        src = src.replace("        prev = cur\n", "        prev = cur\n        first = cur if first is None else first\n", 1)
    mod = types.ModuleType(f"oracle_mutant_{name}")
    mod.__file__ = O.__file__
    exec(compile(src.replace(old, new), f"oracle_mutant_{name}.py", "exec"), mod.__dict__)
    mod.lib, mod.OraShape = O.lib, O.OraShape  # the loaded library and its argument types
    return mod


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_planted_python_mistake_is_caught(name, monkeypatch):
    mod = _py_mutant_module(name)
    monkeypatch.setattr(O, "stream_decode", mod.stream_decode)
    with pytest.raises(AssertionError):
        PIN_FOR_MUTANT[name]()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    tmp = tempfile.mkdtemp(prefix="ora_mut_")
    saved = O._lib
    try:
        so = _mutant_lib(tmp, name)
        O._lib = None
        real, real_build = O._LIB_PATH, O.build
        O._LIB_PATH = so
        O.build = lambda force=False, _so=so: _so  # do not rebuild the real one over the mutant
        try:
            with pytest.raises(AssertionError):
                PIN_FOR_MUTANT[name]()
        finally:
            O._LIB_PATH, O.build = real, real_build
    finally:
        O._lib = saved
        shutil.rmtree(tmp, ignore_errors=True)


# --------------------------------------------------------------------------- quantised label slab
@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
def test_quantized_label_codes_properties(dtype):
    """Codes are integers in [-127, 127] (0 past seq_len), scale * code is within
    scale / 2 of the stored value, the largest |K| of a channel maps to +-127,
    and an all-zero channel has scale 0 and codes 0."""
    sh = Sh(batch=2, n_q_heads=4, n_kv_heads=2, ctx=64, block_size=8, d_qk=16, n_label=8, dtype=dtype, slab_bits=8)
    q, K, V, sl = rand_inputs(sh, 5, dtype=dtype, seq_lens=[64, 37])
    label = np.array([0, 3, 5, 6, 9, 11, 12, 15], np.int32)
    if dtype == W.F32:
        K[:, :, :, 6] = 0.0  # label channel 3: all zero
    else:
        K[:, :, :, 6] = 0
    s = O.shape_of(sh)
    codes, scales = O.quantize_labels(s, K, sl, label)
    Kf = f64(K, dtype)
    for b in range(sh.batch):
        L = int(sl[b])
        assert (codes[b, :, L:] == 0).all()
        for g in range(sh.n_kv_heads):
            for c, ch in enumerate(label):
                col = Kf[b, g, :L, ch]
                sc = float(scales[b, g, c])
                if np.abs(col).max() == 0:
                    assert sc == 0 and (codes[b, g, :L, c] == 0).all()
                    continue
                cd = codes[b, g, :L, c].astype(np.float64)
                assert np.abs(cd).max() == 127 and abs(cd[np.abs(col).argmax()]) == 127
                assert (np.abs(sc * cd - col) <= 0.5 * sc * (1 + 1e-6) + 1e-30).all()


def test_quantized_token_scores_within_the_quantization_bound():
    sh = Sh(batch=2, n_q_heads=8, n_kv_heads=2, ctx=96, block_size=8, d_qk=16, n_label=8, k_b=6, k_t=20)
    q, K, V, sl = rand_inputs(sh, 9, seq_lens=[96, 61])
    label = np.array([1, 2, 4, 7, 8, 10, 13, 14], np.int32)
    s = O.shape_of(sh)
    s8 = O.shape_of(Sh(**{**sh.__dict__, "slab_bits": 8}))
    bidx = O.select_blocks(s, O.block_scores(s, q, O.build_meta(s, K, sl), sl), sl)
    exact, tok = O.token_scores(s, q, K, label, bidx, sl)
    quant, tok8 = O.token_scores(s8, q, K, label, bidx, sl)
    np.testing.assert_array_equal(tok, tok8)
    _, scales = O.quantize_labels(s8, K, sl, label)
    qf = f64(q, W.F32).reshape(sh.batch, sh.n_kv_heads, 4, sh.d_qk)[..., label]  # [B][H][G][r]
    bound = (np.abs(qf).sum(axis=2) * scales * 0.5).sum(axis=-1)  # [B][H]
    ok = tok >= 0
    diff = np.where(ok, np.abs(quant - exact), 0)
    assert (diff <= bound[:, :, None] * (1 + 1e-6)).all()
    assert diff.max() > 0  # the variant does change the scores


def test_quantized_token_scores_exact_on_a_power_of_two_grid():
    """K values m * 2^-3 with integer |m| <= 127 and 127 reached in every label
    channel: scale = 2^-3 exactly, codes = m, scores equal the exact ones."""
    sh = Sh(batch=1, n_q_heads=2, n_kv_heads=1, ctx=32, block_size=8, d_qk=8, n_label=4, k_b=4, k_t=10)
    rng = np.random.default_rng(3)
    m = rng.integers(-127, 128, size=(1, 1, 32, 8)).astype(np.float32)
    m[0, 0, 5, :] = 127.0
    K = (m / 8.0).astype(np.float32)
    q = rng.standard_normal((1, 2, 8)).astype(np.float32)
    sl = np.array([32], np.int32)
    label = np.array([0, 2, 5, 7], np.int32)
    s = O.shape_of(sh)
    s8 = O.shape_of(Sh(**{**sh.__dict__, "slab_bits": 8}))
    codes, scales = O.quantize_labels(s8, K, sl, label)
    assert (scales == np.float32(0.125)).all()
    np.testing.assert_array_equal(codes[0, 0, :, :], m[0, 0][:, label].astype(np.int8))
    bidx = np.array([[[0, 1, 2, 3]]], np.int32)
    exact, _ = O.token_scores(s, q, K, label, bidx, sl)
    quant, _ = O.token_scores(s8, q, K, label, bidx, sl)
    np.testing.assert_array_equal(quant, exact)
