"""The workspace-free block selection (tls_block_score_topk_noalloc).

It exists for callers that may not allocate device memory and have no spare
device buffer to lend the library (for instance code running inside another
runtime's launch hook): their block scores live in a fixed array inside the
library.  This file checks, through the C ABI, that two calls in a row give the
same block selection as the regular entry point with a caller workspace, and
that shapes beyond the array's capacity are refused.  It sits last in the
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
    T.tls_block_score_topk(g.shape, g.q, g.meta, g.seq_lens, ref, None, g.ws)
    torch.cuda.synchronize()
    ref = ref.cpu().numpy()
    for call in range(2):
        got = torch.full((w.batch, w.n_kv_heads, w.k_b), -7, dtype=torch.int32, device="cuda")
        T.tls_block_score_topk_noalloc(g.shape, g.q, g.meta, g.seq_lens, got)
        torch.cuda.synchronize()
        # integer output: bit-exact (the tests' rule for index work)
        np.testing.assert_array_equal(got.cpu().numpy(), ref, err_msg=f"call {call + 1}")


def test_noalloc_rejects_shapes_beyond_the_builtin_array():
    from two_level_sparse_quest_b200 import tls as T

    # 64 sequences * 8 KV heads * 3072 blocks = 1.57 M scores > 1 M
    s = T.make_shape(batch=64, n_q_heads=32, n_kv_heads=8, d_qk=128, d_v=128, block_size=32, n_label=16,
                     k_b=256, k_t=4096, max_ctx=98304, kv_dtype=T.TLS_BF16)
    with pytest.raises(T.TlsError) as e:
        T.tls_block_score_topk_noalloc(s, 256, 256, 256, 256)
    assert e.value.status == T.TLS_ERR_UNSUPPORTED
    assert "built-in array holds 1048576" in str(e.value)
