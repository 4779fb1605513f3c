"""tls_append_tokens: incremental upkeep of the block summary and label slab.

After the K rows of tokens [old, new) are written, the call must leave the
summary and the slab exactly as a full tls_build_block_meta at the new
lengths does (max / min are exact), and as the fp64 oracle's summary of the
same rows.  Cases: one token inside a block, a range crossing a block
boundary, a sequence growing from empty, a multi-block range, ragged
per-sequence ranges, fp32 and bf16, and an invalid range (left untouched, bit
4 of the device error word set).
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


CASES = {
    "bf16_one_token": (W.WORKLOADS["gqa48k_bf16"].with_(batch=2, ctx=4096), [1000, 4000], [1001, 4001], 1),
    "bf16_cross_block": (W.WORKLOADS["gqa48k_bf16"].with_(batch=2, ctx=4096), [1023, 31], [1025, 33], 2),
    "bf16_from_empty": (W.WORKLOADS["gqa48k_bf16"].with_(batch=2, ctx=4096), [0, 0], [37, 1], 37),
    "bf16_multi_block_ragged": (W.WORKLOADS["gqa48k_bf16"].with_(batch=3, ctx=4096), [500, 4000, 64],
                                [700, 4096, 64], 256),
    "f32_ragged": (W.WORKLOADS["tiny_gqa4k_f32"].with_(batch=3, ctx=1000), [0, 999, 400], [5, 1000, 513], 113),
    "bs16_odd": (W.WORKLOADS["gqa48k_bf16"].with_(batch=1, block_size=16, ctx=1999), [1990], [1999], 9),
}


def build(T, g, w, lens):
    edt = torch.int16 if w.dtype == W.BF16 else torch.float32
    meta = torch.zeros((w.batch, w.n_kv_heads, w.n_blocks, 2, w.d_qk), dtype=edt, device="cuda")
    slab = torch.zeros((w.batch, w.n_kv_heads, w.ctx, w.n_label), dtype=edt, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    T.tls_build_block_meta(g.shape, g.K, sl, g.label, meta, slab)
    return meta, slab


@pytest.mark.parametrize("name", sorted(CASES))
def test_append_equals_rebuild_and_oracle(name):
    from oracle import oracle as O
    from tests import _parity as P
    from two_level_sparse_quest_b200 import tls as T

    w, old, new, max_append = CASES[name]
    inp = W.make_decode_inputs(w)
    g = P.GpuInputs(w, inp)
    meta, slab = build(T, g, w, old)
    T.tls_append_tokens(g.shape, g.K, torch.tensor(old, dtype=torch.int32, device="cuda"),
                        torch.tensor(new, dtype=torch.int32, device="cuda"), max_append, g.label, meta, slab)
    ref_meta, ref_slab = build(T, g, w, new)
    torch.cuda.synchronize()
    assert T.tls_device_error(clear=True) == 0
    # bit-exact against a full rebuild at the new lengths (untouched blocks stay 0 in both)
    assert torch.equal(meta.view(torch.int16) if meta.dtype == torch.int16 else meta.view(torch.int32),
                       ref_meta.view(torch.int16) if ref_meta.dtype == torch.int16 else ref_meta.view(torch.int32))
    assert torch.equal(slab, ref_slab)
    # and against the oracle's summary of the same rows
    s = O.shape_of(w)
    om = O.build_meta(s, inp.K, np.asarray(new, np.int32))
    gm = P.from_dev_elems(meta, w.dtype)
    for b in range(w.batch):
        nb = -(-new[b] // w.block_size)
        np.testing.assert_array_equal(gm[b, :, :nb], om[b, :, :nb])


def test_append_rejects_invalid_range_on_device():
    from tests import _parity as P
    from two_level_sparse_quest_b200 import tls as T

    w = W.WORKLOADS["gqa48k_bf16"].with_(batch=2, ctx=1024)
    inp = W.make_decode_inputs(w)
    g = P.GpuInputs(w, inp)
    meta, slab = build(T, g, w, [500, 600])
    m0, s0 = meta.clone(), slab.clone()
    T.tls_device_error(clear=True)
    # sequence 0: new < old; sequence 1: longer than max_append
    T.tls_append_tokens(g.shape, g.K, torch.tensor([500, 600], dtype=torch.int32, device="cuda"),
                        torch.tensor([499, 700], dtype=torch.int32, device="cuda"), 8, g.label, meta, slab)
    torch.cuda.synchronize()
    assert T.tls_device_error(clear=True) == 4
    assert torch.equal(meta, m0) and torch.equal(slab, s0)
