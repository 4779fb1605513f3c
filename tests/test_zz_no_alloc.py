"""The workspace-free block selection (tls_block_score_topk_noalloc).

It exists for callers that may not allocate device memory and have no spare
device buffer to lend the library (for instance code running inside another
runtime's launch hook): their block scores live in a fixed array inside the
library.  This file checks, through the C ABI, that two calls in a row give the
same block selection as the regular entry point with a caller workspace, that
the fp32 block scores left in the built-in array (read back with
tls_noalloc_read_scores) are the regular call's block_score_out bit for bit,
and that shapes beyond the array's capacity are refused.  It sits last in the
collection order so that a failure here leaves every other test already run.
"""
import numpy as np
import pytest
import torch

from two_level_sparse_quest_b200 import workloads as W

pytestmark = pytest.mark.gpu

CASES = {
    "gqa96k_b8_bf16": W.WORKLOADS["gqa96k_b8_bf16"].with_(ctx=16384),
    "gqa48k_bf16": W.WORKLOADS["gqa48k_bf16"],
    "tiny_gqa4k_f32_ragged": W.WORKLOADS["tiny_gqa4k_f32"].with_(batch=3),
    # the latent shape (one KV head shared by 64 query heads, 576 channels)
    "mla64k_b4_bf16_ctx16k": W.WORKLOADS["mla64k_b4_bf16"].with_(ctx=16384),
    # the max-over-heads variant writes the same score layout
    "gqa48k_bf16_agg_max": W.WORKLOADS["gqa48k_bf16"].with_(block_agg=1),
}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from two_level_sparse_quest_b200 import build

    build.build()


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_selection_matches_workspace_entry_point_twice(name):
    from tests import _parity as P
    from two_level_sparse_quest_b200 import tls as T

    w = CASES[name]
    sl = [w.ctx - 37 * b for b in range(w.batch)]
    inp = W.make_decode_inputs(w, seq_lens=sl)
    g = P.GpuInputs(w, inp)
    ref = torch.full((w.batch, w.n_kv_heads, w.k_b), -7, dtype=torch.int32, device="cuda")
    ref_sc = torch.zeros((w.batch, w.n_kv_heads, w.n_blocks), dtype=torch.float32, device="cuda")
    T.tls_block_score_topk(g.shape, g.q, g.meta, g.seq_lens, ref, ref_sc, g.ws)
    torch.cuda.synchronize()
    ref = ref.cpu().numpy()
    ref_sc = ref_sc.cpu().numpy()
    n_scores = ref_sc.size
    for call in range(2):
        got = torch.full((w.batch, w.n_kv_heads, w.k_b), -7, dtype=torch.int32, device="cuda")
        T.tls_block_score_topk_noalloc(g.shape, g.q, g.meta, g.seq_lens, got)
        sc = torch.full((n_scores,), float("nan"), dtype=torch.float32, device="cuda")
        T.tls_noalloc_read_scores(sc, n_scores)
        torch.cuda.synchronize()
        # integer output: bit-exact (the tests' rule for index work)
        np.testing.assert_array_equal(got.cpu().numpy(), ref, err_msg=f"call {call + 1}")
        # the same kernel computes both score arrays: identical bits
        np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), ref_sc.reshape(-1).view(np.uint32),
                                      err_msg=f"scores, call {call + 1}")
    assert T.tls_device_error(clear=True) == 0


def test_noalloc_rejects_shapes_beyond_the_builtin_array():
    from two_level_sparse_quest_b200 import tls as T

    # 64 sequences * 8 KV heads * 3072 blocks = 1.57 M scores > 1 M
    s = T.make_shape(batch=64, n_q_heads=32, n_kv_heads=8, d_qk=128, d_v=128, block_size=32, n_label=16,
                     k_b=256, k_t=4096, max_ctx=98304, kv_dtype=T.TLS_BF16)
    with pytest.raises(T.TlsError) as e:
        T.tls_block_score_topk_noalloc(s, 256, 256, 256, 256)
    assert e.value.status == T.TLS_ERR_UNSUPPORTED
    assert "built-in array holds 1048576" in str(e.value)
