"""tls_select_step (stages 1-4 in one launch) against the two separate calls.

The fused launch runs the same arithmetic as tls_block_score_topk followed by
tls_token_score_topk, so every output must be identical bit for bit: block
ids, token ids, and both score arrays.  The separate calls are themselves
checked against the fp64 oracle in test_gpu_parity.py.  Cases cover ragged and
empty sequences, partial blocks, clamped K_b / K_t, fp32 and bf16, latent
attention shapes, tie-heavy keys and the benchmark's full size.
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


def periodic(w, period_blocks, seq_lens=None):
    inp = W.make_decode_inputs(w, seq_lens=seq_lens)
    t = np.arange(w.ctx) % (period_blocks * w.block_size)
    inp.K = np.ascontiguousarray(inp.K[:, :, t])
    return inp


CASES = {
    "f32_ragged_empty": (W.WORKLOADS["tiny_gqa4k_f32"].with_(batch=4, ctx=512, k_b=4, k_t=40), [0, 1, 31, 512], None),
    "bf16_small": (W.WORKLOADS["gqa48k_bf16"].with_(batch=2, ctx=4096, k_b=24, k_t=300), [4096, 4001], None),
    "bf16_bs16_odd": (W.WORKLOADS["gqa48k_bf16"].with_(block_size=16, ctx=1999, k_b=40, k_t=333), None, None),
    "clamp_kb": (W.WORKLOADS["gqa48k_bf16"].with_(ctx=200, k_b=64, k_t=50), [200], None),
    "mla_small": (W.WORKLOADS["mla64k_b4_bf16"].with_(batch=2, ctx=4096, k_b=16, k_t=300, n_needles=4),
                  [4096, 3000], None),
    "ties_bf16": (W.WORKLOADS["gqa48k_bf16"].with_(batch=2, ctx=4096, k_b=24, k_t=300), [4096, 3999], 5),
    "ties_kmax": (W.WORKLOADS["gqa48k_bf16"].with_(batch=1, ctx=32768, k_b=512, k_t=5000), None, 7),
    "full_gqa96k_b8": (W.WORKLOADS["gqa96k_b8_bf16"], None, None),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_select_step_equals_separate_calls(name):
    from tests import _parity as P
    from two_level_sparse_quest_b200 import tls as T

    w, sl, period = CASES[name]
    inp = periodic(w, period, sl) if period else W.make_decode_inputs(w, seq_lens=sl)
    g = P.GpuInputs(w, inp)
    bidx, bsc = g.block_stage()
    tidx, tsc = g.token_stage(bidx)
    fb = torch.full_like(bidx, -7)
    ft = torch.full_like(tidx, -7)
    fbs = torch.zeros_like(bsc)
    fts = torch.zeros_like(tsc)
    T.tls_select_step(g.shape, g.q, g.meta, g.slab, g.label, g.seq_lens, fb, ft, fbs, fts)
    torch.cuda.synchronize()
    assert T.tls_device_error(clear=True) == 0
    assert torch.equal(fb, bidx), "block ids differ"
    assert torch.equal(ft, tidx), "token ids differ"
    assert torch.equal(fbs.view(torch.int32), bsc.view(torch.int32)), "block scores differ"
    assert torch.equal(fts.view(torch.int32), tsc.view(torch.int32)), "token scores differ"
    # and without the optional score outputs
    fb2 = torch.full_like(bidx, -7)
    ft2 = torch.full_like(tidx, -7)
    T.tls_select_step(g.shape, g.q, g.meta, g.slab, g.label, g.seq_lens, fb2, ft2)
    torch.cuda.synchronize()
    assert torch.equal(fb2, bidx) and torch.equal(ft2, tidx)
