"""GPU parity: every stage of the CUDA path against the fp64 oracle (B200).

Small cases span several tiles and ragged tails and cover the edge cases
(ragged and empty sequences, partial last blocks, k_b >= number of blocks,
k_t >= candidates, group sizes 1/2/4/8, bf16 output).  The five named
workloads run at their full sizes, in the launch configuration the benchmark
uses.  Comparison rules are in tests/_parity.py.
"""
import numpy as np
import pytest
import torch

from two_level_sparse_quest_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from two_level_sparse_quest_b200 import build

    build.build()


def P():
    from tests import _parity

    return _parity


SMALL = {
    "tiny_f32_ragged": (W.WORKLOADS["tiny_gqa4k_f32"].with_(batch=3, ctx=1000, k_b=8, k_t=100), [1000, 777, 33]),
    "gqa_bf16_small": (W.WORKLOADS["gqa48k_bf16"].with_(batch=2, ctx=4096, k_b=24, k_t=300), [4096, 4001]),
    "gqa_bf16_g8": (W.WORKLOADS["gqa48k_bf16"].with_(n_q_heads=64, ctx=2048, k_b=16, k_t=257), None),
    "gqa_bf16_g1": (W.WORKLOADS["gqa48k_bf16"].with_(n_q_heads=8, ctx=2048, k_b=16, k_t=130), None),
    "gqa_bf16_g2_d64": (W.WORKLOADS["gqa48k_bf16"].with_(n_q_heads=16, d_qk=64, d_v=64, ctx=3000, k_b=20,
                                                        k_t=200, n_outlier=4), None),
    "gqa_f32_d128": (W.WORKLOADS["tiny_gqa4k_f32"].with_(batch=2, d_qk=128, d_v=128, n_kv_heads=2, n_q_heads=8, ctx=2500,
                                                         k_b=10, k_t=96), [2500, 1501]),
    "clamp_kb_ge_nblocks": (W.WORKLOADS["gqa48k_bf16"].with_(ctx=200, k_b=64, k_t=50), [200]),
    "clamp_kt_ge_candidates": (W.WORKLOADS["gqa48k_bf16"].with_(ctx=1024, k_b=4, k_t=500), [1024]),
    "empty_and_tiny_sequences": (W.WORKLOADS["tiny_gqa4k_f32"].with_(batch=4, ctx=512, k_b=4, k_t=40),
                                 [0, 1, 31, 512]),
    "block_size_16_odd_ctx": (W.WORKLOADS["gqa48k_bf16"].with_(block_size=16, ctx=1999, k_b=40, k_t=333), None),
    "mla_small": (W.WORKLOADS["mla64k_b4_bf16"].with_(batch=2, ctx=4096, k_b=16, k_t=300, n_needles=4),
                  [4096, 3000]),
    # latent shapes with 16 and 32 heads, and a batch whose CTA ranges of
    # 32-token tiles cross group boundaries (35 tiles per group, 2 per CTA)
    "mla_g16": (W.WORKLOADS["mla64k_b4_bf16"].with_(batch=3, n_q_heads=16, ctx=4096, k_b=16, k_t=300, n_needles=4),
                [4096, 2100, 0]),
    "mla_g32": (W.WORKLOADS["mla64k_b4_bf16"].with_(batch=2, n_q_heads=32, ctx=4096, k_b=16, k_t=300, n_needles=4),
                [3001, 4096]),
    "mla_ranges_cross_groups": (W.WORKLOADS["mla64k_b4_bf16"].with_(batch=6, ctx=8192, k_b=24, k_t=1100, n_needles=8),
                                [8192, 5000, 33, 8192, 1, 7000]),
    # 16 tiles of 32 tokens per group, one per CTA, and a second sequence
    # whose short length leaves most of its CTAs without a valid token
    "mla_one_tile_per_cta": (W.WORKLOADS["mla64k_b4_bf16"].with_(batch=2, ctx=4096, k_b=16, k_t=512, n_needles=4),
                             [4096, 200]),
    # shape sweep: MHA (one query head per KV head) and MQA (one KV head for
    # 16, 32 or 64 query heads: units of 16 heads on the warp-MMA kernel)
    "mha_h16": (W.WORKLOADS["gqa48k_bf16"].with_(n_q_heads=16, n_kv_heads=16, ctx=2048, k_b=16, k_t=200), None),
    "mqa_g16": (W.WORKLOADS["gqa48k_bf16"].with_(batch=2, n_q_heads=16, n_kv_heads=1, ctx=4096, k_b=24, k_t=300),
                [4096, 2999]),
    "mqa_g32": (W.WORKLOADS["gqa48k_bf16"].with_(batch=2, n_q_heads=32, n_kv_heads=1, ctx=4096, k_b=24, k_t=300),
                [4096, 1777]),
    "mqa_g64_d64": (W.WORKLOADS["gqa48k_bf16"].with_(batch=3, n_q_heads=64, n_kv_heads=1, d_qk=64, d_v=64, ctx=3000,
                                                     k_b=20, k_t=211), [3000, 17, 2500]),
    "mqa_g32_f32": (W.WORKLOADS["tiny_gqa4k_f32"].with_(batch=2, n_q_heads=32, n_kv_heads=1, ctx=1000, k_b=8,
                                                        k_t=100), [1000, 640]),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_parity(name):
    w, sl = SMALL[name]
    res = P().full_stage_parity(w, seq_lens=sl, name=name)
    assert res["chained_groups_identical"] >= 0


def sharpened(inp, factor):
    """The same inputs with every bf16 query multiplied by a power of two
    (exact): the block and token rankings do not change, the softmax becomes
    sharper, and a head's running max grows by many log2 units across tiles."""
    q = (inp.q.astype(np.uint32) << 16).view(np.float32) * np.float32(factor)
    inp.q = (q.view(np.uint32) >> 16).astype(np.uint16)
    return inp


@pytest.mark.parametrize("name,factor", [("mla_ranges_cross_groups", 16.0), ("mla_small", 64.0),
                                         ("mla_one_tile_per_cta", 64.0)])
def test_latent_attention_sharp_softmax(name, factor):
    """Large score spreads: the latent kernel's reference max moves and the
    running output is rescaled inside a CTA's range."""
    w, sl = SMALL[name]
    inp = sharpened(W.make_decode_inputs(w, seq_lens=sl), factor)
    P().full_stage_parity(w, inp=inp, name=f"{name}:x{factor:g}")


def test_bf16_output_parity():
    w = W.WORKLOADS["gqa48k_bf16"].with_(ctx=4096, k_b=24, k_t=300)
    P().full_stage_parity(w, out_dtype=W.BF16, name="bf16_out")


def test_full_selection_equals_full_attention_gpu():
    # K_b = all blocks, K_t = all tokens: the sparse step is dense attention
    w = W.WORKLOADS["gqa48k_bf16"].with_(ctx=2048, k_b=64, k_t=2048)
    P().full_stage_parity(w, name="full_selection")


def periodic_keys(w, period_blocks, seq_lens=None):
    """Seeded inputs whose keys repeat every `period_blocks` blocks: block
    summaries, block scores and label-channel token scores then repeat exactly,
    so both top-k boundaries fall inside long runs of equal scores and the
    lower-id rule decides which of them are kept."""
    inp = W.make_decode_inputs(w, seq_lens=seq_lens)
    P_tok = period_blocks * w.block_size
    t = np.arange(w.ctx) % P_tok
    inp.K = np.ascontiguousarray(inp.K[:, :, t])
    return inp


TIES = {
    # 26 copies of the top block score for k_b = 24; each token score 24 times for k_t = 300
    "ties_bf16": (W.WORKLOADS["gqa48k_bf16"].with_(batch=2, ctx=4096, k_b=24, k_t=300), 5, [4096, 3999]),
    "ties_f32_ragged": (W.WORKLOADS["tiny_gqa4k_f32"].with_(batch=3, ctx=1000, k_b=8, k_t=100), 3, [1000, 777, 33]),
    # the token boundary cuts a run at the largest candidate count (16384)
    "ties_bf16_kmax": (W.WORKLOADS["gqa48k_bf16"].with_(batch=1, ctx=32768, k_b=512, k_t=5000), 7, None),
}


@pytest.mark.parametrize("name", sorted(TIES))
def test_tie_heavy_selection_parity(name):
    w, period, sl = TIES[name]
    inp = periodic_keys(w, period, seq_lens=sl)
    P().full_stage_parity(w, name=name, inp=inp)


AGG_MAX = {
    # the max-over-heads block aggregation variant, through the separate stages
    "agg_max_bf16_g4": (W.WORKLOADS["gqa48k_bf16"].with_(batch=2, ctx=4096, k_b=24, k_t=300, block_agg=1),
                        [4096, 3001]),
    "agg_max_f32_ragged": (W.WORKLOADS["tiny_gqa4k_f32"].with_(batch=3, ctx=1000, k_b=8, k_t=100, n_q_heads=8,
                                                                block_agg=1), [1000, 777, 33]),
    "agg_max_full_gqa96k_b8": (W.WORKLOADS["gqa96k_b8_bf16"].with_(block_agg=1), None),
    # more heads per group than the CUDA-core variant takes: the per-head bounds as a tcgen05 GEMM
    "agg_max_bf16_g16": (W.WORKLOADS["gqa48k_bf16"].with_(batch=2, n_q_heads=32, n_kv_heads=2, ctx=4096, k_b=24,
                                                          k_t=300, block_agg=1), [4096, 2900]),
    "agg_max_bf16_mqa_g32": (W.WORKLOADS["gqa48k_bf16"].with_(batch=2, n_q_heads=32, n_kv_heads=1, ctx=4096, k_b=24,
                                                              k_t=300, block_agg=1), [4096, 1777]),
    "agg_max_bf16_mqa_g64_d64": (W.WORKLOADS["gqa48k_bf16"].with_(batch=3, n_q_heads=64, n_kv_heads=1, d_qk=64,
                                                                  d_v=64, ctx=3000, k_b=20, k_t=211, block_agg=1),
                                 [3000, 17, 2500]),
    "agg_max_mla_small": (W.WORKLOADS["mla64k_b4_bf16"].with_(batch=2, ctx=4096, k_b=16, k_t=300, n_needles=4,
                                                              block_agg=1), [4096, 3000]),
    "agg_max_full_mla64k_b4": (W.WORKLOADS["mla64k_b4_bf16"].with_(block_agg=1), None),
}


@pytest.mark.parametrize("name", sorted(AGG_MAX))
def test_max_aggregation_variant_parity(name):
    w, sl = AGG_MAX[name]
    res = P().full_stage_parity(w, seq_lens=sl, name=name)
    assert res["block_swaps"] <= max(1, res["groups"] // 8)


def test_max_aggregation_select_step_equals_separate_calls():
    from tests import _parity as PP
    from two_level_sparse_quest_b200 import tls as T

    w = W.WORKLOADS["gqa48k_bf16"].with_(batch=2, ctx=4096, k_b=24, k_t=300, block_agg=1)
    g = PP.GpuInputs(w, W.make_decode_inputs(w))
    bidx, _ = g.block_stage()
    tidx, _ = g.token_stage(bidx)
    fb, ft = torch.full_like(bidx, -7), torch.full_like(tidx, -7)
    T.tls_select_step(g.shape, g.q, g.meta, g.slab, g.label, g.seq_lens, fb, ft)
    torch.cuda.synchronize()
    assert torch.equal(fb, bidx) and torch.equal(ft, tidx)


FULL = ["tiny_gqa4k_f32", "gqa48k_bf16", "gqa96k_b8_bf16", "mla64k_b4_bf16"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_parity(name):
    res = P().full_stage_parity(W.WORKLOADS[name], name=f"full:{name}")
    # index sets bit-exact except counted boundary swaps
    assert res["block_swaps"] <= max(1, res["groups"] // 8)
    assert res["token_swaps"] <= max(1, res["groups"] // 8)


@pytest.mark.parametrize("impl", ["cuda_core", "tensor_core", "warp_mma"])
def test_alternative_attention_kernels_parity(impl):
    """The attention kernels that TLS_ATTN_IMPL selects instead of the default
    (read once per process, so each runs in a child process): the CUDA-core
    kernel for GQA bf16 and latent shapes, the tcgen05 kernel for GQA bf16,
    the warp-MMA latent kernel for latent shapes."""
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cases = {"cuda_core": ["gqa_bf16_small", "gqa_bf16_g8", "mla_small", "mqa_g32", "mqa_g64_d64"],
             "tensor_core": ["gqa_bf16_small", "gqa_bf16_g8"],
             "warp_mma": ["mla_small", "mla_g16", "mla_g32"]}[impl]
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "from tests import test_gpu_parity as t, _parity as P\n"
        "for n in %r:\n"
        "    w, sl = t.SMALL[n]\n"
        "    P.full_stage_parity(w, seq_lens=sl, name=n + ':' + %r)\n"
        "print('ok')\n" % (root, cases, impl))
    env = dict(os.environ, TLS_ATTN_IMPL=impl)
    r = subprocess.run([sys.executable, "-c", code], env=env, cwd=root, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-4000:]


SLAB_Q8 = {
    # the int8 label slab: codes and scales bit-exact, token scores and
    # selections against the oracle's quantised reading
    "q8_r16_ragged": (W.WORKLOADS["gqa48k_bf16"].with_(batch=2, ctx=4096, k_b=24, k_t=300, slab_bits=8),
                      [4096, 3001]),
    "q8_r32_g8": (W.WORKLOADS["gqa48k_bf16"].with_(n_q_heads=64, ctx=2048, k_b=16, k_t=257, n_label=32,
                                                   slab_bits=8), None),
    "q8_r64_d64_empty": (W.WORKLOADS["gqa48k_bf16"].with_(batch=4, n_q_heads=16, d_qk=64, d_v=64, ctx=512, k_b=4,
                                                          k_t=40, n_label=64, slab_bits=8), [0, 1, 31, 512]),
    "q8_mla_small": (W.WORKLOADS["mla64k_b4_bf16"].with_(batch=2, ctx=4096, k_b=16, k_t=300, n_needles=4,
                                                         slab_bits=8), [4096, 3000]),
    "q8_full_gqa96k_b8": (W.WORKLOADS["gqa96k_b8_bf16"].with_(slab_bits=8), None),
}


@pytest.mark.parametrize("name", sorted(SLAB_Q8))
def test_int8_label_slab_parity(name):
    w, sl = SLAB_Q8[name]
    res = P().full_stage_parity(w, seq_lens=sl, name=name)
    assert res["token_swaps"] <= max(1, res["groups"] // 8)


def test_int8_label_slab_select_step_equals_separate_calls():
    from tests import _parity as PP
    from two_level_sparse_quest_b200 import tls as T

    w = W.WORKLOADS["gqa48k_bf16"].with_(batch=2, ctx=4096, k_b=24, k_t=300, slab_bits=8)
    g = PP.GpuInputs(w, W.make_decode_inputs(w, seq_lens=[4096, 2222]))
    bidx, _ = g.block_stage()
    tidx, _ = g.token_stage(bidx)
    fb, ft = torch.full_like(bidx, -7), torch.full_like(tidx, -7)
    T.tls_select_step(g.shape, g.q, g.meta, g.slab, g.label, g.seq_lens, fb, ft)
    torch.cuda.synchronize()
    assert torch.equal(fb, bidx) and torch.equal(ft, tidx)
